"""Pins of the CPU oracle against facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself: code points
published in the OCP FP8 and bfloat16 formats (cross-checked with torch's own
converters), closed forms, special cases that reduce to a library routine,
invariants of the definitions, and the hand-worked examples in
tests/golden/hand_examples.json.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


HAND = _load("hand_examples.json")


def bits_of(ids, N):
    dense = np.zeros(N, dtype=bool)
    dense[list(ids)] = True
    return synth.pack_bits(dense)[0]


# --------------------------------------------------------------------- decoders
def test_bf16_code_points():
    assert oracle.decode_bf16(0x3F80) == 1.0
    assert oracle.decode_bf16(0xBF80) == -1.0
    assert oracle.decode_bf16(0x0001) == 2.0 ** -133          # smallest subnormal
    assert oracle.decode_bf16(0x0080) == 2.0 ** -126          # smallest normal
    assert oracle.decode_bf16(0x7F7F) == (2 - 2 ** -7) * 2.0 ** 127
    assert math.isinf(oracle.decode_bf16(0x7F80))
    assert math.isnan(oracle.decode_bf16(0x7FC0))
    # every code against torch's bfloat16 -> float32 conversion
    codes = np.arange(1 << 16, dtype=np.uint16)
    ref = torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).float().numpy().astype(np.float64)
    got = oracle.decode_rows(codes.reshape(-1, 64)).ravel()
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


def test_e4m3_code_points():
    # OCP 8-bit floating point specification, E4M3: bias 7, max 448, NaN S.1111.111
    assert oracle.decode_e4m3(0x7E) == 448.0
    assert oracle.decode_e4m3(0xFE) == -448.0
    assert math.isnan(oracle.decode_e4m3(0x7F)) and math.isnan(oracle.decode_e4m3(0xFF))
    assert oracle.decode_e4m3(0x78) == 256.0                  # exponent 15 is finite
    assert oracle.decode_e4m3(0x38) == 1.0
    assert oracle.decode_e4m3(0x08) == 2.0 ** -6              # smallest normal
    assert oracle.decode_e4m3(0x01) == 2.0 ** -9              # smallest subnormal
    assert oracle.decode_e4m3(0x07) == 7 * 2.0 ** -9          # largest subnormal
    assert oracle.decode_e4m3(0x00) == 0.0
    assert math.copysign(1.0, oracle.decode_e4m3(0x80)) == -1.0
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    got = np.array([oracle.decode_e4m3(c) for c in codes])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


def test_e8m0_code_points():
    assert oracle.decode_e8m0(127) == 1.0
    assert oracle.decode_e8m0(0) == 2.0 ** -127
    assert oracle.decode_e8m0(254) == 2.0 ** 127
    assert math.isnan(oracle.decode_e8m0(255))


def test_fp8_rows_decode_blockwise():
    """A stored FP8 row is [E4M3 * 2^(scale-127) per 64-block | bf16 RoPE]."""
    g = np.random.default_rng(5)
    x = g.standard_normal((6, 512)) * np.exp2(g.integers(-8, 8, size=(6, 1)))
    kv = synth.encode_rows(x, "e4m3")
    dec = oracle.decode_rows(kv)
    e4 = torch.from_numpy(kv.data).view(torch.float8_e4m3fn).double().numpy()
    sc = np.exp2(kv.scale.astype(np.float64) - 127.0)
    ref_nope = e4 * np.repeat(sc, 64, axis=1)
    ref_rope = torch.from_numpy(kv.rope.view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.array_equal(dec[:, :448], ref_nope)
    assert np.array_equal(dec[:, 448:], ref_rope)
    # the encoding keeps each value within half an E4M3 step (2^-4 relative,
    # or half the 2^-9 subnormal step of the scaled block)
    s64 = np.repeat(sc, 64, axis=1)
    err = np.abs(dec[:, :448] - x[:, :448])
    assert np.all(err <= 2.0 ** -4 * np.abs(x[:, :448]) + 2.0 ** -10 * s64)


# ----------------------------------------------------------------- index score
def _score_inputs(seed, H, N, dtype="bf16"):
    g = np.random.default_rng(seed)
    q = g.standard_normal((H, 128)) / math.sqrt(128)
    k = g.standard_normal((N, 128)) / math.sqrt(128)
    w = g.random(H).astype(np.float32)
    qs = synth.bf16_bits(q) if dtype != "f32" else q.astype(np.float32)
    keys = synth.encode_rows(k, dtype)
    return qs, w, keys


@pytest.mark.parametrize("dtype", ["f32", "bf16", "e4m3"])
def test_score_one_hot_weight_is_relu_dot(dtype):
    """w = e_h reduces the score to max(q_h . k_j, 0): a library dot product."""
    H, N = 8, 300
    q, w, keys = _score_inputs(1, H, N, dtype)
    qd = oracle.decode_rows(q.reshape(H, 128))
    kd = oracle.decode_rows(keys)
    for h in (0, 3, 7):
        e = np.zeros(H, dtype=np.float32)
        e[h] = 1.0
        s = oracle.index_score(q[None], e[None], keys, 1, 1, H, N)[0, 0]
        ref = np.maximum(kd @ qd[h], 0.0).astype(np.float32)
        np.testing.assert_allclose(s, ref, rtol=1e-6, atol=1e-7)


def test_score_linear_in_head_weights():
    """s(w) = sum_h w_h s(e_h): the heads combine linearly through w."""
    H, N = 8, 257
    q, w, keys = _score_inputs(2, H, N)
    full = oracle.index_score(q[None], w[None], keys, 1, 1, H, N)[0, 0].astype(np.float64)
    parts = np.zeros(N)
    for h in range(H):
        e = np.zeros(H, dtype=np.float32)
        e[h] = 1.0
        parts += float(w[h]) * oracle.index_score(q[None], e[None], keys, 1, 1, H, N)[0, 0]
    np.testing.assert_allclose(full, parts, rtol=3e-7, atol=1e-7)


def test_score_all_negative_dots_is_zero_and_cond():
    H, N = 4, 64
    g = np.random.default_rng(3)
    k = np.abs(g.standard_normal((N, 128)))
    q = -np.abs(g.standard_normal((H, 128)))
    keys = synth.encode_rows(k, "f32")
    w = np.ones(H, dtype=np.float32)
    s, cond, mag = oracle.index_score(q.astype(np.float32)[None], w[None], keys, 1, 1, H, N, want_cond=True,
                                      want_mag=True)
    assert np.all(s == 0.0)
    # every dot is negative: |q_h . k| = sum_d |q_hd k_d| = -(q_h . k), so both
    # tolerance terms equal the score of -q
    s2 = oracle.index_score((-q).astype(np.float32)[None], w[None], keys, 1, 1, H, N)
    np.testing.assert_allclose(cond[0, 0], s2[0, 0], rtol=1e-6)
    np.testing.assert_allclose(mag[0, 0], s2[0, 0], rtol=1e-6)


@pytest.mark.parametrize("ex", HAND["score"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_score_signed_weight_hand_examples(ex, dtype):
    """Signed head weights multiply the ReLU of each head's dot product (the
    weight sits outside the ReLU).  Key k = e_0 and q_h = dot_h e_0 give the
    dots exactly; the expected scores were worked by hand."""
    w = np.array(ex["w"], dtype=np.float32)
    H = len(w)
    q = np.zeros((H, 128))
    q[:, 0] = ex["q_dot_k"]
    k = np.zeros((3, 128))
    k[:, 0] = 1.0
    k[1, 0] = 2.0  # entry 1 doubles every dot, and the score with it
    qs = synth.bf16_bits(q) if dtype == "bf16" else q.astype(np.float32)
    s, cond = oracle.index_score(qs[None], w[None], synth.encode_rows(k, dtype), 1, 1, H, 3, want_cond=True)
    assert s[0, 0, 0] == ex["score"] and s[0, 0, 2] == ex["score"]
    assert s[0, 0, 1] == 2 * ex["score"]
    assert cond[0, 0, 0] == sum(abs(a) * abs(b) for a, b in zip(ex["w"], ex["q_dot_k"]))


def test_score_batch_and_query_indexing():
    """Entry (b, t, j) only sees query (b, t) and key (b, j)."""
    B, Q, H, N = 2, 3, 4, 40
    g = np.random.default_rng(4)
    q = g.standard_normal((B, Q, H, 128)).astype(np.float32)
    w = g.random((B, Q, H)).astype(np.float32)
    k = g.standard_normal((B * N, 128))
    keys = synth.encode_rows(k, "f32")
    s = oracle.index_score(q, w, keys, B, Q, H, N)
    for b in range(B):
        for t in range(Q):
            one = oracle.index_score(q[b, t][None], w[b, t][None], keys.slice(b * N, (b + 1) * N),
                                     1, 1, H, N)[0, 0]
            assert np.array_equal(s[b, t], one)


def test_planted_rows_are_the_topk():
    """The +3 sigma planted rows of the 128K batched workload dominate the noise
    (planted scores ~8 vs noise ~1.1 +- 0.24), so the top-k is the planted set."""
    spec = synth.scaled(synth.DECODE_128K_B32, B=2, N=2048, k=64)
    inp = synth.decode_layer(spec)
    for b in range(spec.B):
        s = oracle.index_score(inp["q_idx"][b][None], inp["w"][b][None],
                               inp["keys"].slice(b * spec.N, (b + 1) * spec.N), 1, 1, spec.H, spec.N)[0, 0]
        ids, n, _ = oracle.topk(s, spec.k)
        assert n == spec.k
        assert np.array_equal(ids, inp["planted"][b])
        gap = np.sort(s)[::-1]
        assert gap[spec.k - 1] > 3.0 * gap[spec.k]


# ----------------------------------------------------------------------- top-k
@pytest.mark.parametrize("ex", HAND["topk"])
def test_topk_hand_examples(ex):
    ids, n, _ = oracle.topk(np.array(ex["scores"], dtype=np.float32), ex["k"])
    assert ids.tolist() == ex["ids"] and n == ex["n_sel"]


@pytest.mark.parametrize("ex", HAND["topk_masked"])
def test_topk_masked_examples(ex):
    ids, n, _ = oracle.topk(np.array(ex["scores"], dtype=np.float32), ex["k"],
                            np.array(ex["allowed"], dtype=np.uint8))
    assert ids.tolist() == ex["ids"] and n == ex["n_sel"]


@pytest.mark.parametrize("kind", ["normal", "ties", "signed", "const"])
@pytest.mark.parametrize("N,k", [(1, 1), (7, 3), (100, 100), (1000, 64), (4096, 512), (300, 1000)])
def test_topk_brute_force(kind, N, k):
    s = synth.random_scores(11, 1, N, kind)[0]
    ids, n, _ = oracle.topk(s, k)
    ref = sorted(range(N), key=lambda j: (-float(s[j]), j))[:k]
    assert n == min(k, N)
    assert ids[:n].tolist() == sorted(ref)
    assert np.all(ids[n:] == -1)
    # invariant: every selected score >= every unselected score
    sel = np.zeros(N, dtype=bool)
    sel[ids[:n]] = True
    if n < N:
        assert s[sel].min() >= s[~sel].max()


def test_topk_nan_is_never_selected():
    s = np.array([1.0, np.nan, 3.0, np.nan, 2.0], dtype=np.float32)
    ids, n, nn = oracle.topk(s, 4)
    assert ids.tolist() == [0, 2, 4, -1] and n == 3 and nn == 2


# ------------------------------------------------------------------- attention
def _rows(g, n, D=512):
    return synth.encode_rows(g.standard_normal((n, D)), "f32")


def test_attn_single_row_returns_the_row():
    g = np.random.default_rng(6)
    kv = _rows(g, 10)
    q = g.standard_normal((4, 512)).astype(np.float32)
    out, lse = oracle.attn(q, kv, 10, np.array([7], dtype=np.int32), scale=0.05)
    assert np.array_equal(out, np.broadcast_to(kv.data[7], out.shape))
    ref = 0.05 * (q.astype(np.float64) @ kv.data[7].astype(np.float64))
    np.testing.assert_allclose(lse, ref, rtol=1e-6)


def test_attn_equal_logits_is_the_mean():
    g = np.random.default_rng(7)
    kv = _rows(g, 20)
    swa = _rows(g, 5)
    q = np.zeros((2, 512), dtype=np.float32)
    ids = np.array([1, 4, 9, -1, -1], dtype=np.int32)
    out, lse = oracle.attn(q, kv, 20, ids, swa=swa, swa_len=5)
    rows = np.concatenate([kv.data[[1, 4, 9]], swa.data]).astype(np.float64)
    np.testing.assert_allclose(out[0], rows.mean(axis=0), rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(lse, np.log(8.0), rtol=1e-7)


def test_attn_matches_library_softmax():
    """Small case against scipy's softmax and numpy matmul on decoded rows."""
    g = np.random.default_rng(8)
    spec = synth.scaled(synth.DECODE_64K, N=300, H=8, swa=16)
    inp = synth.decode_layer(spec)
    ids = np.sort(g.choice(300, 40, replace=False)).astype(np.int32)
    out, lse = oracle.attn(inp["q_attn"][0], inp["kv"], 300, ids, swa=inp["swa"], swa_len=16,
                           scale=spec.scale)
    X = np.concatenate([oracle.decode_rows(inp["kv"])[ids], oracle.decode_rows(inp["swa"])])
    qd = oracle.decode_rows(inp["q_attn"][0])
    logits = spec.scale * qd @ X.T
    ref = scipy.special.softmax(logits, axis=1) @ X
    np.testing.assert_allclose(out, ref, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(lse, scipy.special.logsumexp(logits, axis=1), rtol=1e-6)


def test_attn_split_merge_identity():
    """Softmax over R1 u R2 equals the lse-weighted merge of the two halves:
    the identity the split-K decode relies on."""
    g = np.random.default_rng(9)
    kv = _rows(g, 64)
    q = g.standard_normal((3, 512)).astype(np.float32)
    ids = np.arange(64, dtype=np.int32)
    o, l = oracle.attn(q, kv, 64, ids, scale=0.04)
    o1, l1 = oracle.attn(q, kv, 64, ids[:25], scale=0.04)
    o2, l2 = oracle.attn(q, kv, 64, ids[25:], scale=0.04)
    L = np.logaddexp(l1.astype(np.float64), l2)
    merged = (np.exp(l1 - L)[:, None] * o1 + np.exp(l2 - L)[:, None] * o2)
    np.testing.assert_allclose(o, merged, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(l, L, rtol=1e-6)


def test_attn_empty_and_padding():
    g = np.random.default_rng(10)
    kv = _rows(g, 8)
    q = g.standard_normal((2, 512)).astype(np.float32)
    out, lse = oracle.attn(q, kv, 8, np.array([-1, -1], dtype=np.int32))
    assert np.all(out == 0) and np.all(np.isneginf(lse))
    with pytest.raises(oracle.OracleError):
        oracle.attn(q, kv, 8, np.array([8], dtype=np.int32))


# ---------------------------------------------------------------------- golden
def test_golden_rows_sum_to_one_and_single_head():
    spec = synth.scaled(synth.EVAL_WINDOW, N=200, T=3, H=4)
    inp = synth.eval_layer(spec, 0)
    p = oracle.golden(inp["qa"], inp["kv"], spec.T, spec.H, spec.N, spec.scale)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=2e-6)
    X = oracle.decode_rows(inp["kv"])
    qd = oracle.decode_rows(inp["qa"].reshape(-1, 512)).reshape(spec.T, spec.H, 512)
    ref = scipy.special.softmax(spec.scale * qd @ X.T, axis=2).mean(axis=1)
    np.testing.assert_allclose(p, ref, rtol=1e-5, atol=1e-9)


def test_golden_agrees_with_attention_lse():
    """p_h(j) = exp(logit_hj - lse_h): the golden probabilities and the
    attention log-sum-exp over all entries describe the same softmax."""
    spec = synth.scaled(synth.EVAL_WINDOW, N=150, T=1, H=1)
    inp = synth.eval_layer(spec, 1)
    p = oracle.golden(inp["qa"], inp["kv"], 1, 1, spec.N, spec.scale)[0]
    _, lse = oracle.attn(inp["qa"][0], inp["kv"], spec.N, np.arange(spec.N, dtype=np.int32),
                         scale=spec.scale)
    X = oracle.decode_rows(inp["kv"])
    logit = spec.scale * X @ oracle.decode_rows(inp["qa"][0])[0]
    np.testing.assert_allclose(p, np.exp(logit - lse[0]), rtol=1e-5)


def test_golden_index_closed_forms():
    """The softmax-of-the-indexer-logits reading: values fixed in closed form
    (a uniform row, logits that differ by ln 3 and ln 2), and the same values
    at logits near 1000, where exp without the row maximum subtracted
    overflows."""
    ln2, ln3 = np.log(2.0), np.log(3.0)
    p = oracle.golden_index(np.array([[2.5] * 8, [0.0, ln3] + [-np.inf] * 6], dtype=np.float32))
    np.testing.assert_array_equal(p[0], np.full(8, 0.125, dtype=np.float32))
    np.testing.assert_allclose(p[1, :2], [0.25, 0.75], rtol=1e-6)
    assert np.all(p[1, 2:] == 0)
    x = np.array([1000.0 + ln2, 1000.0, 1000.0], dtype=np.float32)
    d = float(x[0]) - 1000.0  # the stored offset (fp32 spacing at 1000 is 6e-5)
    p = oracle.golden_index(x)
    np.testing.assert_allclose(p, np.array([np.exp(d), 1.0, 1.0]) / (np.exp(d) + 2.0), rtol=1e-6)
    assert abs(p[0] - 0.5) < 1e-4


def test_golden_index_nan_and_empty_rows():
    """NaN and -inf logits carry no mass; a row with no finite logit is all
    zeros; otherwise a row sums to 1 and matches scipy's softmax over its
    finite entries."""
    g = np.random.default_rng(5)
    s = g.standard_normal((3, 300)).astype(np.float32) * 4
    s[1, ::7] = np.nan
    s[1, 3::11] = -np.inf
    s[2, :] = -np.inf
    p = oracle.golden_index(s)
    assert np.all(p[2] == 0)
    fin = np.isfinite(s[1])
    assert np.all(p[1, ~fin] == 0)
    np.testing.assert_allclose(p[1, fin], scipy.special.softmax(s[1, fin].astype(np.float64)), rtol=1e-6)
    np.testing.assert_allclose(p[0], scipy.special.softmax(s[0].astype(np.float64)), rtol=1e-6)
    np.testing.assert_allclose(p[:2].sum(axis=1), 1.0, rtol=1e-6)


# ----------------------------------------------------------------------- top-p
@pytest.mark.parametrize("ex", HAND["topp"])
def test_topp_hand_examples(ex):
    bits, n = oracle.topp(np.array(ex["p"], dtype=np.float32))
    assert synth.unpack_bits(bits, len(ex["p"]))[0].nonzero()[0].tolist() == ex["set"]
    assert n == len(ex["set"])


@pytest.mark.parametrize("conc", [0.5, 2.0, 6.0])
def test_topp_minimal_prefix_invariants(conc):
    N = 3000
    p = synth.random_probs(12, 1, N, conc)[0]
    bits, n = oracle.topp(p)
    sel = synth.unpack_bits(bits, N)[0]
    m = np.floor(p.astype(np.float64) * 2.0 ** oracle.TOPP_SHIFT).astype(np.uint64)
    M = int(m.sum(dtype=np.uint64))
    T = -(-M * 3 // 5)
    mass = int(m[sel].sum(dtype=np.uint64))
    assert mass >= T
    # prefix of the ranking (descending p, ties to lower index)
    order = sorted(range(N), key=lambda j: (-float(p[j]), j))
    assert set(order[:n]) == set(np.nonzero(sel)[0].tolist())
    # minimal: without its last-ranked member the set falls short
    assert mass - int(m[order[n - 1]]) < T


# ------------------------------------------------------------------------ vote
@pytest.mark.parametrize("ex", HAND["vote"])
def test_vote_hand_examples(ex):
    N, L, j = 40, 21, 17
    sets = np.zeros((L, 2), dtype=np.uint32)
    for l in ex["layers_selecting"]:
        sets[l] = bits_of([j], N)
    out = oracle.vote(sets, N, 3)
    assert bool(synth.unpack_bits(out, N)[0][j]) == ex["kept"]


def test_vote_and_union_against_counts():
    N, L = 1000, 21
    sets = synth.random_bits(13, L, N, 0.1)
    dense = synth.unpack_bits(sets, N)
    out = synth.unpack_bits(oracle.vote(sets, N, 3), N)[0]
    assert np.array_equal(out, dense.sum(axis=0) >= 3)
    u = synth.unpack_bits(oracle.union(sets[:5], N), N)[0]
    assert np.array_equal(u, dense[:5].any(axis=0))
    # padding bits beyond N stay clear
    assert oracle.vote(sets, N, 0)[-1] >> (N % 32) == 0


# ------------------------------------------------------------------------- LSA
@pytest.mark.parametrize("ex", HAND["lsa"])
def test_lsa_hand_examples(ex):
    out = oracle.lsa_gate(np.array([[ex["logit"]]], dtype=np.float32))
    assert bool(out[0] & 1) == ex["fetched"]


def test_lsa_nonnegative_weights_fetch_everything():
    """With every u_h >= 0 and beta = 0 the logit sum_h u_h ReLU(.) is never
    negative, so every entry passes sigmoid >= 0.5 (a degenerate gate)."""
    H, N = 6, 500
    q, _, keys = _score_inputs(14, H, N)
    u = np.random.default_rng(14).random(H).astype(np.float32)
    logit = oracle.index_score(q[None], u[None], keys, 1, 1, H, N)[0]
    assert synth.unpack_bits(oracle.lsa_gate(logit), N)[0].all()


def test_lsa_or_over_layers():
    a = np.array([-1.0, 2.0, -3.0, -0.5], dtype=np.float32)
    b = np.array([-1.0, -2.0, 0.5, -0.5], dtype=np.float32)
    out = synth.unpack_bits(oracle.lsa_gate(np.stack([a, b]), beta=0.25), 4)[0]
    assert out.tolist() == [False, True, True, False]


# --------------------------------------------------------------------- overlap
@pytest.mark.parametrize("ex", HAND["overlap"])
def test_overlap_hand_examples(ex):
    c = oracle.overlap(bits_of(ex["a"], ex["N"]), bits_of(ex["b"], ex["N"]), ex["N"])
    assert list(c) == ex["counts"]


def test_overlap_random_baseline_matches_page():
    """Two independent random k-subsets of N overlap in k^2/N on average, so
    the reported fraction |A&B|/k has mean k/N: keep 512 of ~800 gives 0.67
    (the page's random baseline; 512/768 = 0.667)."""
    facts = _load("page_facts.json")["random_overlap_keep512_of_800"]
    k, N = facts["k"], 768
    g = np.random.default_rng(15)
    fr = []
    for _ in range(400):
        a = bits_of(g.choice(N, k, replace=False), N)
        b = bits_of(g.choice(N, k, replace=False), N)
        both, na, nb = oracle.overlap(a, b, N)
        assert na == nb == k
        fr.append(both / k)
    fr = np.array(fr)
    se = fr.std(ddof=1) / math.sqrt(len(fr))
    assert abs(fr.mean() - k / N) < 3 * se + 1e-12
    assert round(fr.mean(), 2) == facts["value"]
    # the Act 1 random baseline 57.6% corresponds to N = 512 / 0.576 ~ 889 chunks
    n_act1 = 512 / _load("page_facts.json")["random_overlap_act1"]["value"]
    assert 880 < n_act1 < 900


# ------------------------------------------------------------ the write side
# The storage format is the architecture post's ("why quantising the KV does
# not save memory", point 1); E4M3 is the OCP E4M3FN format it names: bias 7,
# 3 mantissa bits, no infinities, S.1111.111 NaN, largest value 448.
def test_e4m3_encode_round_trips_every_code():
    for c in range(256):
        if c & 0x7F == 0x7F:
            continue  # the two NaN codes
        assert oracle.encode_e4m3(oracle.decode_e4m3(c)) == c, hex(c)


def test_e4m3_encode_ties_to_even_and_rounds_to_nearest():
    """Between two adjacent codes the midpoint goes to the even code (mantissa
    LSB 0, which is the code's LSB), anything off the midpoint to the nearer."""
    for c in range(0x7E):
        lo, hi = oracle.decode_e4m3(c), oracle.decode_e4m3(c + 1)
        mid = (lo + hi) / 2
        assert oracle.encode_e4m3(mid) == (c if c % 2 == 0 else c + 1), hex(c)
        assert oracle.encode_e4m3(mid - (hi - lo) * 1e-3) == c
        assert oracle.encode_e4m3(mid + (hi - lo) * 1e-3) == c + 1
        assert oracle.encode_e4m3(-mid) == 0x80 | (c if c % 2 == 0 else c + 1)


@pytest.mark.parametrize("v,code", [(448.0, 0x7E), (464.0, 0x7E), (1e9, 0x7E), (float("inf"), 0x7E),
                                    (-float("inf"), 0xFE), (float("nan"), 0x7F), (2.0 ** -6, 0x08),
                                    (7 * 2.0 ** -9, 0x07), (2.0 ** -9, 0x01), (2.0 ** -10, 0x00),
                                    (-0.0, 0x80), (1.0, 0x38), (-1.75, 0xBE)])
def test_e4m3_encode_code_points(v, code):
    """OCP E4M3FN code points: 448 = 0x7E is the largest value and larger
    magnitudes saturate to it; 2^-6 = 0x08 is the smallest normal, 2^-9 = 0x01
    the smallest subnormal."""
    assert oracle.encode_e4m3(v) == code


def test_e4m3_encode_matches_torch_float8():
    """A library routine for in-range values: torch's float8_e4m3fn cast
    (round to nearest even)."""
    g = np.random.default_rng(40)
    v = np.concatenate([g.standard_normal(4000) * 100, g.standard_normal(2000) * 2.0 ** -7,
                        g.uniform(-448, 448, 2000)]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.encode_e4m3(float(x)) for x in v], dtype=np.uint8)
    inr = np.abs(v) <= 448
    assert np.array_equal(got[inr], ref[inr])


def test_block_scale_is_the_finest_that_fits():
    """The stored scale 2^e is the smallest power of two with amax <= 448 * 2^e
    (an all-zero block takes e = 0)."""
    for amax, code in [(448.0, 127), (449.0, 128), (224.0, 126), (224.0001, 127), (0.0, 127), (1.0, 119)]:
        assert oracle.e8m0_for(amax) == code, amax
    g = np.random.default_rng(41)
    for a in np.exp(g.uniform(-80, 80, 500)):
        e = oracle.e8m0_for(a) - 127
        assert a <= 448 * 2.0 ** e and a > 448 * 2.0 ** (e - 1)


def test_bf16_encode_ties_to_even_and_matches_torch():
    assert oracle.encode_bf16(1.0 + 2.0 ** -8) == 0x3F80      # midpoint of 1.0 and 1+2^-7: even
    assert oracle.encode_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82  # midpoint of 1+2^-7 and 1+2^-6: even
    assert oracle.encode_bf16(float(np.float32(3.0e38))) == 0x7F62  # 0x7F61B1E6 rounds up
    assert oracle.encode_bf16(float(np.float32(3.4e38))) == 0x7F80  # past the largest bf16: inf
    g = np.random.default_rng(42)
    v = (g.standard_normal(5000) * np.exp(g.uniform(-30, 30, 5000))).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.encode_bf16(float(x)) for x in v], dtype=np.uint16)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("dim", [128, 512])
def test_encode_rows_decodes_within_half_a_step(dim):
    """Decoding an encoded row returns each value within half an E4M3 step
    of its binade times the block scale; each block's largest magnitude lands
    in (224, 448] after scaling; RoPE dims within bf16 rounding."""
    g = np.random.default_rng(43)
    x = (g.standard_normal((6, dim)) * np.exp(g.uniform(-20, 20, (6, dim // 64)).repeat(64, axis=1))).astype(
        np.float32)
    enc = oracle.encode_rows(x, "e4m3")
    assert enc["finite"]
    kv = synth.KV("e4m3", dim, enc["data"], enc["scale"], enc["rope"])
    dec = oracle.decode_rows(kv)
    nope = dim - 64
    sc = np.exp2(enc["scale"].astype(np.float64) - 127).repeat(64, axis=1)
    xs = np.abs(x[:, :nope]).astype(np.float64)
    assert np.all(np.abs(dec[:, :nope] - x[:, :nope]) <= 2.0 ** -4 * xs + 2.0 ** -10 * sc)
    amax = xs.reshape(6, -1, 64).max(axis=2) / sc[:, ::64]
    assert np.all((amax > 224) & (amax <= 448))
    assert np.all(np.abs(dec[:, nope:] - x[:, nope:]) <= 2.0 ** -8 * np.abs(x[:, nope:]))
