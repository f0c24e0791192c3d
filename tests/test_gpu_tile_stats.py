"""GPU parity of the score bounds (scorer side output, top-k input).

The record is defined in include/lidx.h (LIDX_STATS_SPAN): per score row and
span of 32 entries, the largest and the smallest order-preserving key of the
span's non-NaN scores.  `bounds_of` writes that definition out on the host:
it builds the top-k's input from scores, and checks the scorer's side output
against the scores the same call produced (a property of the call).  Every
selection is compared with the oracle's top-k on the same fp32 scores."""
import numpy as np
import pytest
import torch

import lightning_indexer_top_index_b200 as L
import oracle
import synth
from _helpers import dev_kv, dev_q

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_device):
    from lightning_indexer_top_index_b200 import build
    build.build()
    yield


def order_keys(s: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(s, dtype=np.float32).view(np.uint32).copy()
    u[u == 0x80000000] = 0  # -0 as +0
    key = np.where((u & 0x80000000) != 0, ~u, u | np.uint32(0x80000000)).astype(np.uint32)
    key[np.isnan(s)] = 0
    return key


def bounds_of(s: np.ndarray) -> np.ndarray:
    """[rows][N] float32 -> [rows][ceil(N/32)][2] uint32 (max key, min key)."""
    rows, N = s.shape
    n = (N + L.STATS_SPAN - 1) // L.STATS_SPAN
    out = np.zeros((rows, n, 2), dtype=np.uint32)
    for r in range(rows):
        k = order_keys(s[r])
        pad = np.zeros(n * L.STATS_SPAN, dtype=np.uint32)
        pad[:N] = k
        spans = pad.reshape(n, L.STATS_SPAN)
        out[r, :, 0] = spans.max(axis=1)
        out[r, :, 1] = np.where(spans == 0, np.uint32(0xFFFFFFFF), spans).min(axis=1)
    return out


def _dev_bounds(b):
    return torch.from_numpy(b.view(np.int32)).cuda()


def _check(s, ids, n_sel, k, allowed=None):
    ids, n_sel = ids.cpu().numpy(), n_sel.cpu().numpy()
    for r in range(s.shape[0]):
        ref_ids, ref_n, _ = oracle.topk(s[r], k, None if allowed is None else allowed[r])
        assert n_sel[r, 0] == ref_n, f"row {r}"
        assert np.array_equal(ids[r, 0], ref_ids), f"row {r}"


@pytest.mark.parametrize("kind", ["normal", "ties", "signed", "const"])
@pytest.mark.parametrize("N,k", [(1, 1), (37, 5), (1024, 64), (16384, 512), (16385, 512), (4000, 4000),
                                 (300, 1000), (60001, 1024)])
def test_topk_from_bounds_bit_exact(kind, N, k):
    s = synth.random_scores(51, 2, N, kind)
    st = torch.from_numpy(s).cuda().reshape(2, 1, N)
    b = _dev_bounds(bounds_of(s)).reshape(2, 1, -1, 2)
    ids, n_sel, _, _ = L.topk_select(st, k, tile_stats=b)
    _check(s, ids, n_sel, k)


def test_topk_bounds_with_nan_and_allowed_mask():
    N = 5000
    s = synth.random_scores(52, 3, N, "ties")
    s[1, ::97] = np.nan
    s[2, :] = np.nan
    s[2, 7] = 1.0
    allowed = (np.random.default_rng(52).random((3, N)) < 0.3).astype(np.uint8)
    allowed[2, 7] = 1
    b = _dev_bounds(bounds_of(s)).reshape(3, 1, -1, 2)
    st = torch.from_numpy(s).cuda().reshape(3, 1, N)
    ids = torch.empty((3, 1, 256), dtype=torch.int32, device="cuda")
    ws = L.workspace(L.workspace_size(L.OP_TOPK, L.topk_args(st, 256, torch.from_numpy(allowed).cuda(), ids)))
    ids, n_sel, _, _ = L.topk_select(st, 256, torch.from_numpy(allowed).cuda(), ws=ws, tile_stats=b)
    _check(s, ids, n_sel, 256, allowed)
    assert L.read_device_status(ws) & L.DEV_NAN
    ids, n_sel, _, _ = L.topk_select(st, 64, tile_stats=b)
    _check(s, ids, n_sel, 64)


def test_topk_wrong_bounds_stay_in_bounds():
    """Bounds that do not hold give wrong ids but no write outside ids[0..k)."""
    N, k = 8000, 256
    s = synth.random_scores(53, 1, N, "normal")
    bogus = bounds_of(s)
    bogus[:, :, 0] = order_keys(np.array([0.5], np.float32))[0]   # claims max 0.5
    bogus[:, :, 1] = order_keys(np.array([0.25], np.float32))[0]  # and min 0.25
    buf = torch.full((k + 64,), 12345, dtype=torch.int32, device="cuda")
    ids = buf[:k].view(1, 1, k)
    L.topk_select(torch.from_numpy(s).cuda().reshape(1, 1, N), k, ids=ids,
                  tile_stats=_dev_bounds(bogus).reshape(1, 1, -1, 2))
    torch.cuda.synchronize()
    assert torch.all(buf[k:] == 12345)


@pytest.mark.parametrize("spec", [
    synth.TINY_1K_F32,
    synth.scaled(synth.DECODE_64K, N=5000),
    synth.scaled(synth.DECODE_64K, N=16384),
    synth.scaled(synth.DECODE_64K, N=3001, B=3, H=32),
    synth.scaled(synth.DECODE_500K_FP8, N=3001, B=2),
], ids=lambda s: f"{s.name}-N{s.N}-B{s.B}-H{s.H}")
def test_scorer_bounds_then_topk(spec):
    """The scorer's bounds describe exactly its own scores; the top-k that
    starts from them equals the oracle's top-k of those scores."""
    inp = synth.decode_layer(spec)
    B, H, N = spec.B, spec.H, spec.N
    keys = dev_kv(inp["keys"], batch_rows=N)
    q = dev_q(inp["q_idx"].reshape(B, 1, H, 128), spec.q_dtype)
    w = torch.from_numpy(inp["w"].reshape(B, 1, H)).cuda()
    n = (N + L.STATS_SPAN - 1) // L.STATS_SPAN
    b = torch.zeros((B, 1, n, 2), dtype=torch.int32, device="cuda")
    scores = L.index_score(q, w, keys, N, tile_stats=b)
    s = scores.cpu().numpy().reshape(B, N)
    assert np.array_equal(b.cpu().numpy().view(np.uint32).reshape(B, n, 2), bounds_of(s))
    ids, n_sel, _, _ = L.topk_select(scores, spec.k, tile_stats=b)
    _check(s, ids, n_sel, spec.k)


def test_scorer_bounds_batched_queries():
    """Several queries per key tile."""
    spec = synth.scaled(synth.EVAL_WINDOW, T=7, N=3000, H=64, L=1)
    inp = synth.eval_layer(spec, 0)
    T, H, N = spec.T, spec.H, spec.N
    keys = dev_kv(inp["keys"], batch_rows=N)
    q = dev_q(inp["q_idx"].reshape(1, T, H, 128), "bf16")
    w = torch.from_numpy(inp["w"].reshape(1, T, H)).cuda()
    n = (N + L.STATS_SPAN - 1) // L.STATS_SPAN
    b = torch.zeros((1, T, n, 2), dtype=torch.int32, device="cuda")
    scores = L.index_score(q, w, keys, N, tile_stats=b)
    s = scores.cpu().numpy().reshape(T, N)
    assert np.array_equal(b.cpu().numpy().view(np.uint32).reshape(T, n, 2), bounds_of(s))
    ids, n_sel, _, _ = L.topk_select(scores.view(T, 1, N), 256, tile_stats=b.view(T, 1, n, 2))
    _check(s, ids, n_sel, 256)
