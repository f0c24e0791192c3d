"""The cache write side (lidx_cache_append) against the oracle's encoder, bit
for bit: new rows are quantised into the storage format (architecture post,
"why quantising the KV does not save memory", point 1: E4M3 with a
power-of-two scale per 64 elements, bf16 RoPE dims) and written at their
positions, linearly or into a ring (the sliding window).  Every byte of the
cache planes is compared, so rows outside the written positions must be
left as they were."""
import numpy as np
import pytest
import torch

import lightning_indexer_top_index_b200 as L
import oracle

pytestmark = pytest.mark.gpu


def _rows(seed, n, dim):
    """fp32 rows whose 64-element blocks span many binades, with the hard
    cases planted: an all-zero block, exact E4M3 midpoints times a power of
    two, values exactly at 448 * 2^e, tiny and negative-zero values."""
    g = np.random.default_rng(seed)
    x = g.standard_normal((n, dim)) * np.exp2(g.integers(-40, 40, (n, dim // 64))).repeat(64, axis=1)
    x = x.astype(np.float32)
    if n >= 4:
        x[0, :64] = 0.0
        mids = np.array([(oracle.decode_e4m3(c) + oracle.decode_e4m3(c + 1)) / 2 for c in range(64)])
        x[1, :64] = (mids * 2.0 ** 5).astype(np.float32)
        x[1, 0] = 448 * 2.0 ** 5  # the block's largest magnitude exactly at 448 * 2^5
        x[2, 64:128] = np.float32(2.0 ** -140)
        x[2, 64] = np.float32(-0.0)
        x[3, :] = -x[3, :]
    return x


def _empty_cache(dtype, dim, rows, seed):
    """A cache of `rows` rows filled with random bytes (so that writes outside
    the target rows would show)."""
    g = np.random.default_rng(seed)
    if dtype == "e4m3":
        data = torch.from_numpy(g.integers(0, 256, (rows, dim - 64), dtype=np.uint8)).cuda()
        scale = torch.from_numpy(g.integers(0, 256, (rows, (dim - 64) // 64), dtype=np.uint8)).cuda()
        rope = torch.from_numpy(g.integers(-2 ** 15, 2 ** 15, (rows, 64), dtype=np.int16)).cuda().view(torch.bfloat16)
        return L.DeviceKV(L.E4M3, dim, data, scale, rope)
    if dtype == "bf16":
        return L.DeviceKV(L.BF16, dim, torch.from_numpy(
            g.integers(-2 ** 15, 2 ** 15, (rows, dim), dtype=np.int16)).cuda().view(torch.bfloat16))
    return L.DeviceKV(L.F32, dim, torch.from_numpy(g.standard_normal((rows, dim)).astype(np.float32)).cuda())


def _planes(kv):
    out = [kv.data.cpu().view(torch.uint8).numpy().copy()]
    if kv.scale is not None:
        out.append(kv.scale.cpu().numpy().copy())
        out.append(kv.rope.cpu().view(torch.uint8).numpy().copy())
    return out


def _expected(before, x, dtype, dim, dest_rows):
    """Apply the oracle's encoding of rows x at the given cache rows."""
    enc = oracle.encode_rows(x, dtype)
    exp = [p.copy() for p in before]
    data = enc["data"].view(np.uint8).reshape(x.shape[0], -1)
    for i, r in enumerate(dest_rows):
        if r is None:
            continue
        exp[0][r] = data[i]
        if dtype == "e4m3":
            exp[1][r] = enc["scale"][i]
            exp[2][r] = enc["rope"][i].view(np.uint8)
    return exp, enc["finite"]


@pytest.mark.parametrize("dtype", ["e4m3", "bf16", "f32"])
@pytest.mark.parametrize("dim", [512, 128])
@pytest.mark.parametrize("ring", [0, 128])
def test_append_bit_exact(cuda_device, dtype, dim, ring):
    B, R, cap = 3, 9, 300
    cache = _empty_cache(dtype, dim, B * cap, 50 + dim + ring)
    cache.batch_rows = cap
    x = _rows(51 + dim, B * R, dim)
    pos = np.array([5, 250, 123], dtype=np.int32) if ring == 0 else np.array([120, 255, 3], dtype=np.int32)
    before = _planes(cache)
    ws = L.cache_append(torch.from_numpy(x.reshape(B, R, dim)).cuda(), cache, torch.from_numpy(pos).cuda(), cap,
                        ring)
    torch.cuda.synchronize()
    dest = []
    for b in range(B):
        for r in range(R):
            p = int(pos[b]) + r
            idx = p % ring if ring else p
            dest.append(b * cap + idx if idx < cap else None)
    exp, finite = _expected(before, x, dtype, dim, dest)
    got = _planes(cache)
    for g_, e_ in zip(got, exp):
        assert np.array_equal(g_, e_)
    assert finite and L.read_device_status(ws) == 0


def test_append_out_of_range_and_nonfinite(cuda_device):
    """A row whose destination lies beyond the capacity is skipped
    (LIDX_DEV_BOUNDS); NaN and infinities are stored as the format says (NaN
    code 0x7F, infinities saturated) and raise LIDX_DEV_NAN."""
    B, R, cap, dim = 2, 4, 10, 512
    cache = _empty_cache("e4m3", dim, B * cap, 60)
    cache.batch_rows = cap
    x = _rows(61, B * R, dim)
    x[1, 3] = np.nan
    x[2, 70] = np.inf
    x[5, 450] = -np.inf  # a RoPE dim: bf16 -inf
    pos = np.array([8, 0], dtype=np.int32)  # rows 10 and 11 of sequence 0 do not exist
    before = _planes(cache)
    ws = L.cache_append(torch.from_numpy(x.reshape(B, R, dim)).cuda(), cache, torch.from_numpy(pos).cuda(), cap)
    torch.cuda.synchronize()
    dest = [8, 9, None, None, cap + 0, cap + 1, cap + 2, cap + 3]
    exp, finite = _expected(before, x, "e4m3", dim, dest)
    assert not finite
    got = _planes(cache)
    for g_, e_ in zip(got, exp):
        assert np.array_equal(g_, e_)
    st = L.read_device_status(ws)
    assert st & L.DEV_BOUNDS and st & L.DEV_NAN


def test_appended_rows_feed_the_attention(cuda_device):
    """Rows appended into an E4M3 cache are read back by the attention as the
    oracle decodes them: attend over exactly the appended rows."""
    B, R, cap, dim = 1, 64, 128, 512
    cache = _empty_cache("e4m3", dim, cap, 70)
    x = np.random.default_rng(71).standard_normal((R, dim)).astype(np.float32)
    L.cache_append(torch.from_numpy(x.reshape(B, R, dim)).cuda(), cache,
                   torch.zeros(1, dtype=torch.int32, device="cuda"), cap)
    g = np.random.default_rng(72)
    q = g.standard_normal((64, dim)).astype(np.float32)
    qb = torch.from_numpy(q).cuda().to(torch.bfloat16)
    ids = torch.arange(R, dtype=torch.int32, device="cuda").reshape(1, R)
    out, _ = L.sparse_attn_decode(qb.reshape(1, 64, dim), cache, cap, ids, None, None, 0, dim ** -0.5)
    import synth
    planes = _planes(cache)
    kv = synth.KV("e4m3", dim, planes[0], planes[1], planes[2].view(np.uint16))
    qbits = qb.cpu().view(torch.int16).numpy().view(np.uint16)
    ro, _ = oracle.attn(qbits, kv, cap, np.arange(R, dtype=np.int32), scale=dim ** -0.5)
    o = out.cpu().numpy()[0]
    rel = np.abs(o - ro).max(axis=-1) / np.abs(ro).max(axis=-1)
    assert rel.max() <= 2e-3
