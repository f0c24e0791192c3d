"""The allocation-free attention entry point, for callers that cannot allocate
device memory when they call (a plugin hosted by another runtime with no
scratch allocator, a serving loop that forbids cudaMalloc after start-up).

It is called through the C ABI, twice in a row on different inputs (the
shared scratch array keeps the previous call's contents), and each result is
checked against lidx_sparse_attn_decode on the same inputs within the
attention tolerance.  The second call must leave the device's free memory
unchanged.  This file is collected last on purpose."""
import ctypes as C

import numpy as np
import pytest
import torch

import lightning_indexer_top_index_b200 as L
import synth
from _helpers import ATTN_TOL, dev_kv, dev_q

pytestmark = pytest.mark.gpu


def _case(spec, layer, seed):
    inp = synth.decode_layer(spec, layer)
    g = np.random.default_rng(seed)
    ids = np.full((spec.B, spec.k), -1, dtype=np.int32)
    for b in range(spec.B):
        m = spec.k - 7 * b
        ids[b, :m] = np.sort(g.choice(spec.N, m, replace=False))
    return (dev_q(inp["q_attn"], "bf16"), dev_kv(inp["kv"], batch_rows=spec.N),
            dev_kv(inp["swa"], batch_rows=spec.swa), torch.from_numpy(ids).cuda())


def test_noalloc_matches_workspace_entry_point(cuda_device):
    from lightning_indexer_top_index_b200 import build
    build.build()
    lib = L.lib()
    fn = lib.lidx_sparse_attn_decode_noalloc
    fn.restype = C.c_int
    fn.argtypes = [C.POINTER(L.AttnArgs), C.c_void_p, C.c_void_p]
    spec = synth.scaled(synth.DECODE_64K, N=3000, B=2, k=256)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call, (layer, seed) in enumerate([(0, 5), (1, 6)]):
        q, kv, swa, ids = _case(spec, layer, seed)
        swa_len = 128 - 50 * call
        ref, ref_lse = L.sparse_attn_decode(q, kv, spec.N, ids, None, swa, swa_len, spec.scale)
        out = torch.full_like(ref, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        a = L.attn_args(q, kv, spec.N, ids, None, swa, swa_len, spec.scale, out, lse)
        st = C.c_void_p(torch.cuda.current_stream().cuda_stream)
        torch.cuda.synchronize()
        free0, torch0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
        assert fn(C.byref(a), C.c_void_p(status.data_ptr()), st) == L.OK
        torch.cuda.synchronize()
        if call > 0:
            # the first call has loaded the library's module (and its array);
            # from then on a call takes no device memory at all
            assert torch.cuda.mem_get_info()[0] == free0, "the call changed the device's free memory"
            assert torch.cuda.memory_allocated() == torch0
        r, o = ref.cpu().numpy().astype(np.float64), out.cpu().numpy().astype(np.float64)
        rel = np.abs(o - r).max(axis=-1) / np.abs(r).max(axis=-1)
        assert rel.max() <= ATTN_TOL, f"call {call}: max relative difference {rel.max():.3e}"
        np.testing.assert_allclose(lse.cpu().numpy(), ref_lse.cpu().numpy(), rtol=1e-5, atol=1e-5)
        assert int(status.item()) == 0


def test_noalloc_rejects_oversized_requests(cuda_device):
    """A request whose split-K scratch exceeds the fixed array is refused
    before anything is enqueued."""
    spec = synth.scaled(synth.DECODE_64K, N=600, B=1, k=512)
    q, kv, swa, ids = _case(spec, 0, 7)
    big_b = 64  # 64 sequences x 20 splits x 64 heads x 514 floats > 16 MiB
    qb = q.expand(big_b, -1, -1).contiguous()
    idb = ids.expand(big_b, -1).contiguous()
    # real per-sequence caches, so the request would also be valid for the workspace entry point
    kvb = L.DeviceKV(kv.dtype, kv.dim, kv.data.repeat(big_b, 1), batch_rows=spec.N)
    swb = L.DeviceKV(swa.dtype, swa.dim, swa.data.repeat(big_b, 1), batch_rows=spec.swa)
    out = torch.empty((big_b, 64, 512), device="cuda")
    a = L.attn_args(qb, kvb, spec.N, idb, None, swb, 128, spec.scale, out, None)
    assert L.workspace_size(L.OP_ATTN, a) > L.NOALLOC_SCRATCH_BYTES
    with pytest.raises(L.LidxError) as e:
        L.sparse_attn_decode_noalloc(qb, kvb, spec.N, idb, None, swb, 128, spec.scale, out=out, want_lse=False)
    assert e.value.status == L.ERR_WORKSPACE
