"""Python binding of liblidx.so: lightning indexer, top-k and sparse MQA decode
for B200 (sm_100a).

Argument marshalling only.  Every step of the path runs in the library's CUDA
kernels; torch supplies device memory and streams.  There is no CPU fallback:
if the library is missing or the device is not sm_100, calls raise.

    import lightning_indexer_top_index_b200 as lidx
    scores = lidx.index_score(q, w, keys)                 # [B][Q][N]
    ids, n_sel = lidx.topk_select(scores, k=512)           # [B][Q][k]
    out, lse = lidx.sparse_attn_decode(q_attn, kv, N, ids[:, 0], n_sel[:, 0], swa, 128, scale)
"""
from __future__ import annotations

import ctypes as C
import dataclasses
import os
import threading
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblidx.so")

# ---------------------------------------------------------------- constants
F32, BF16, E4M3, F16 = 0, 1, 2, 3
DTYPES = {"f32": F32, "bf16": BF16, "e4m3": E4M3, "f16": F16}

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_WORKSPACE = 0, 1, 2, 3, 4
DEV_BOUNDS, DEV_NAN, DEV_TIMEOUT = 0x1, 0x2, 0x4
LAUNCH_PDL = 0x1
LAUNCH_TEST_LOST_ARRIVAL = 0x80000000
STATS_SPAN = 32  # entries per score-bounds record (optional scorer output, top-k input)

EVAL_GOLDEN, EVAL_TOPP, EVAL_VOTE, EVAL_LSA, EVAL_OVERLAP = 0x1, 0x2, 0x4, 0x8, 0x10
EVAL_GOLDEN_INDEX = 0x20  # probs as the softmax of the indexer logits (the other golden reading)
OP_SCORE, OP_TOPK, OP_ATTN, OP_EVAL, OP_DECODE, OP_APPEND = 0, 1, 2, 3, 4, 5

# Layer schedule of DeepSeek-V4-Flash (architecture post, section (A) table):
# layers 0-1 sliding window only, even layers 2..42 CSA (4:1 + top-k), odd
# layers 3..41 HCA (128:1, read densely).
CSA_LAYERS = tuple(range(2, 43, 2))
HCA_LAYERS = tuple(range(3, 42, 2))
GATE_MODEL_LAYERS = (10, 12, 20)  # memory-indexer gate layers (deep-dive write-up, section 4.1)


def csa_stack_index(model_layer: int) -> int:
    """Position of a CSA model layer in the stack of CSA layers."""
    if model_layer not in CSA_LAYERS:
        raise ValueError(f"layer {model_layer} is not a CSA layer")
    return CSA_LAYERS.index(model_layer)


GATE_LAYERS = tuple(csa_stack_index(l) for l in GATE_MODEL_LAYERS)
MODEL_LAYERS = 43
SWA_ROWS = 128


def logical_kv_bytes(tokens: int, elem_bytes: int = 4) -> dict:
    """Logical KV-cache size of the 43-layer stack at a context of `tokens`
    (architecture post, section (A)), `elem_bytes` per element:

      CSA  per layer tokens/4 entries, each a 512-wide attention row and a
           128-d index key
      HCA  per layer tokens/128 entries of a 512-wide row (no index keys)
      SWA  a 128-row window of 512-wide rows in every layer

    The post's ~871 MiB at 64K comes out with 4-byte elements, the logical
    (host-side) cache it names; the stored FP8 rows are smaller."""
    csa = len(CSA_LAYERS) * (tokens // 4) * (512 + 128) * elem_bytes
    hca = len(HCA_LAYERS) * (tokens // 128) * 512 * elem_bytes
    swa = MODEL_LAYERS * min(SWA_ROWS, tokens) * 512 * elem_bytes
    return {"csa": csa, "hca": hca, "swa": swa, "total": csa + hca + swa}


class LidxError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})" if what else status_string(status))


# ---------------------------------------------------------------- ctypes ABI
class KVArgs(C.Structure):
    _fields_ = [("dtype", C.c_int32), ("dim", C.c_int32), ("data", C.c_void_p), ("scale", C.c_void_p),
                ("rope", C.c_void_p), ("ld", C.c_int64), ("ld_scale", C.c_int64), ("ld_rope", C.c_int64),
                ("batch_rows", C.c_int64)]


class ScoreArgs(C.Structure):
    _fields_ = [("B", C.c_int32), ("Q", C.c_int32), ("H", C.c_int32), ("N", C.c_int32),
                ("q_dtype", C.c_int32), ("q", C.c_void_p), ("w", C.c_void_p), ("keys", KVArgs),
                ("scores", C.c_void_p), ("ld_scores", C.c_int64), ("flags", C.c_uint32), ("tile_stats", C.c_void_p),
                ("n_visible", C.c_void_p)]


class TopkArgs(C.Structure):
    _fields_ = [("B", C.c_int32), ("Q", C.c_int32), ("N", C.c_int32), ("k", C.c_int32),
                ("scores", C.c_void_p), ("ld_scores", C.c_int64), ("allowed", C.c_void_p),
                ("ld_allowed", C.c_int64), ("ids", C.c_void_p), ("n_sel", C.c_void_p), ("mask", C.c_void_p),
                ("mask_bits", C.c_void_p), ("flags", C.c_uint32), ("tile_stats", C.c_void_p),
                ("allowed_bits", C.c_void_p), ("ld_allowed_bits", C.c_int64), ("n_valid", C.c_void_p)]


class AttnArgs(C.Structure):
    _fields_ = [("B", C.c_int32), ("H", C.c_int32), ("q_dtype", C.c_int32), ("q", C.c_void_p),
                ("kv", KVArgs), ("N", C.c_int32), ("ids", C.c_void_p), ("n_ids", C.c_int32),
                ("ld_ids", C.c_int64), ("n_sel", C.c_void_p), ("swa", KVArgs), ("swa_len", C.c_int32),
                ("scale", C.c_float), ("out", C.c_void_p), ("lse", C.c_void_p), ("flags", C.c_uint32)]


class EvalArgs(C.Structure):
    _fields_ = [("ops", C.c_uint32), ("L", C.c_int32), ("T", C.c_int32), ("H", C.c_int32), ("N", C.c_int32),
                ("qa_dtype", C.c_int32), ("qa", C.c_void_p), ("kv", KVArgs), ("scale", C.c_float),
                ("probs", C.c_void_p), ("top_p_num", C.c_uint32), ("top_p_den", C.c_uint32),
                ("topp_bits", C.c_void_p), ("min_votes", C.c_int32), ("vote_bits", C.c_void_p),
                ("window_bits", C.c_void_p), ("n_gate", C.c_int32), ("gate_logits", C.c_void_p),
                ("gate_bias", C.c_float), ("fetched_bits", C.c_void_p), ("n_pairs", C.c_int32),
                ("set_a", C.c_void_p), ("ld_a", C.c_int64), ("set_b", C.c_void_p), ("ld_b", C.c_int64),
                ("counts", C.c_void_p), ("index_scores", C.c_void_p), ("ld_index_scores", C.c_int64)]


class DecodeArgs(C.Structure):
    _fields_ = [("B", C.c_int32), ("H", C.c_int32), ("N", C.c_int32), ("k", C.c_int32),
                ("q_idx", C.c_void_p), ("w", C.c_void_p), ("keys", KVArgs), ("H_attn", C.c_int32),
                ("q_attn", C.c_void_p), ("kv", KVArgs), ("swa", KVArgs), ("swa_len", C.c_int32),
                ("scale", C.c_float), ("out", C.c_void_p), ("lse", C.c_void_p), ("scores", C.c_void_p),
                ("ld_scores", C.c_int64), ("ids", C.c_void_p), ("n_sel", C.c_void_p),
                ("prefetch", C.c_void_p * 2), ("prefetch_bytes", C.c_uint64 * 2), ("flags", C.c_uint32)]


class AppendArgs(C.Structure):
    _fields_ = [("B", C.c_int32), ("R", C.c_int32), ("x", C.c_void_p), ("cache", KVArgs),
                ("capacity", C.c_int64), ("pos", C.c_void_p), ("ring", C.c_int32), ("flags", C.c_uint32)]


_STRUCTS = [KVArgs, ScoreArgs, TopkArgs, AttnArgs, EvalArgs, DecodeArgs, AppendArgs]
EXPORTS = ("lidx_index_score", "lidx_topk_select", "lidx_sparse_attn_decode", "lidx_selection_eval",
           "lidx_decode_layer", "lidx_cache_append", "lidx_workspace_size", "lidx_launch_count",
           "lidx_read_device_status",
           "lidx_status_string", "lidx_abi_version", "lidx_struct_size")

_lib = None
_lock = threading.Lock()


def lib():
    """Load liblidx.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"{LIB_PATH} is missing: build it with "
                                  "`python -m lightning_indexer_top_index_b200.build`")
            l = C.CDLL(LIB_PATH)
            P, I, SZ = C.c_void_p, C.c_int, C.c_size_t
            for name, res, args in [
                ("lidx_index_score", I, [C.POINTER(ScoreArgs), P]),
                ("lidx_topk_select", I, [C.POINTER(TopkArgs), P, SZ, P]),
                ("lidx_sparse_attn_decode", I, [C.POINTER(AttnArgs), P, SZ, P]),
                ("lidx_selection_eval", I, [C.POINTER(EvalArgs), P, SZ, P]),
                ("lidx_decode_layer", I, [C.POINTER(DecodeArgs), P, SZ, P]),
                ("lidx_cache_append", I, [C.POINTER(AppendArgs), P, SZ, P]),
                ("lidx_workspace_size", I, [I, P, C.POINTER(SZ)]),
                ("lidx_launch_count", I, [I, P, C.POINTER(I)]),
                ("lidx_read_device_status", I, [P, C.POINTER(C.c_uint32), P]),
                ("lidx_status_string", C.c_char_p, [I]),
                ("lidx_abi_version", I, []),
                ("lidx_struct_size", SZ, [I]),
            ]:
                f = getattr(l, name)
                f.restype = res
                f.argtypes = args
            for i, s in enumerate(_STRUCTS):
                if l.lidx_struct_size(i) != C.sizeof(s):
                    raise ImportError(f"ABI mismatch for {s.__name__}: library {l.lidx_struct_size(i)} "
                                      f"bytes, binding {C.sizeof(s)}")
            _lib = l
    return _lib


def status_string(s: int) -> str:
    return lib().lidx_status_string(int(s)).decode()


def _check(rc: int, what: str):
    if rc != OK:
        raise LidxError(rc, what)


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


# ---------------------------------------------------------------- device rows
@dataclasses.dataclass
class DeviceKV:
    """Device-resident rows in one of the storage formats (see lidx_kv).

    data:  f32 [rows][ld] | bf16 [rows][ld] | uint8 [rows][ld] (E4M3 codes)
    scale: uint8 [rows][ld_scale] E8M0 codes (E4M3 only)
    rope:  bf16 [rows][ld_rope] (E4M3 only)
    """
    dtype: int
    dim: int
    data: torch.Tensor
    scale: Optional[torch.Tensor] = None
    rope: Optional[torch.Tensor] = None
    batch_rows: int = 0

    @staticmethod
    def from_arrays(dtype, dim, data, scale=None, rope=None, batch_rows=0, device="cuda"):
        """Copy host arrays (numpy or torch; bf16 given as uint16 bits) to the device."""
        def dev(x, bf16=False):
            if x is None:
                return None
            t = torch.as_tensor(x)
            if bf16 and t.dtype in (torch.uint16, torch.int16):
                t = t.view(torch.int16).view(torch.bfloat16)
            return t.to(device, non_blocking=False).contiguous()
        dt = DTYPES[dtype] if isinstance(dtype, str) else dtype
        return DeviceKV(dt, dim, dev(data, bf16=dt == BF16), dev(scale), dev(rope, bf16=True), batch_rows)

    def args(self) -> KVArgs:
        ld = self.data.stride(0)
        return KVArgs(self.dtype, self.dim, self.data.data_ptr(), _ptr(self.scale), _ptr(self.rope), ld,
                      0 if self.scale is None else self.scale.stride(0),
                      0 if self.rope is None else self.rope.stride(0), self.batch_rows)

    @property
    def rows(self) -> int:
        return self.data.shape[0]

    def nbytes(self) -> int:
        n = self.data.numel() * self.data.element_size()
        for t in (self.scale, self.rope):
            if t is not None:
                n += t.numel() * t.element_size()
        return n


def _qdtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"query dtype {t.dtype} (expected float32 or bfloat16)")


# ---------------------------------------------------------------- the calls
def index_score(q: torch.Tensor, w: torch.Tensor, keys: DeviceKV, N: int, scores: torch.Tensor = None,
                stream=None, tile_stats: torch.Tensor = None, n_visible: torch.Tensor = None) -> torch.Tensor:
    """scores[b,t,j] = sum_h w[b,t,h] * max(q[b,t,h] . keys[b,j], 0).

    q [B][Q][H][128] (float32 or bfloat16), w [B][Q][H] float32 -> scores
    float32 [B][Q][N] (or the given tensor with a row stride >= N).  With
    `tile_stats` (int32 [B][Q][ceil(N/STATS_SPAN)][2]) the call also writes
    the score bounds topk_select can start from.  `n_visible` (int32 [B][Q])
    is the causal entry mask of prefill queries: entries j >= n_visible[b][t]
    score -inf."""
    B, Q, H, D = q.shape
    assert q.is_contiguous() and w.is_contiguous() and w.dtype == torch.float32
    if scores is None:
        scores = torch.empty((B, Q, N), dtype=torch.float32, device=q.device)
    a = ScoreArgs(B, Q, H, N, _qdtype(q), q.data_ptr(), w.data_ptr(), keys.args(), scores.data_ptr(),
                  scores.stride(1), 0, _ptr(tile_stats), _ptr(n_visible))
    _check(lib().lidx_index_score(C.byref(a), _stream(stream)), "lidx_index_score")
    return scores


def workspace_size(op: int, args) -> int:
    n = C.c_size_t(0)
    _check(lib().lidx_workspace_size(op, C.byref(args), C.byref(n)), "lidx_workspace_size")
    return n.value


def launch_count(op: int, args) -> int:
    """Kernels the call `op` launches for `args` on the current device."""
    n = C.c_int(0)
    _check(lib().lidx_launch_count(op, C.byref(args), C.byref(n)), "lidx_launch_count")
    return n.value


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A zeroed, 256-byte aligned workspace tensor (the status word starts clear)."""
    return torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)


def topk_args(scores, k, allowed=None, ids=None, n_sel=None, mask=None, mask_bits=None, flags=0,
              tile_stats=None, allowed_bits=None, n_valid=None) -> TopkArgs:
    B, Q, N = scores.shape[0], scores.shape[1], scores.shape[2]
    ldb = 0 if allowed_bits is None else (allowed_bits.stride(0) if allowed_bits.dim() > 1 else (N + 31) // 32)
    return TopkArgs(B, Q, N, k, scores.data_ptr(), scores.stride(1), _ptr(allowed),
                    0 if allowed is None else allowed.stride(0), _ptr(ids), _ptr(n_sel), _ptr(mask),
                    _ptr(mask_bits), flags, _ptr(tile_stats), _ptr(allowed_bits), ldb, _ptr(n_valid))


def topk_select(scores: torch.Tensor, k: int, allowed: torch.Tensor = None, *, want_mask=False,
                want_bits=False, ids=None, n_sel=None, ws=None, stream=None, tile_stats=None, bits=None,
                allowed_bits: torch.Tensor = None, n_valid: torch.Tensor = None):
    """Top-k row ids of scores [B][Q][N] (N = scores.shape[2]).

    Returns (ids int32 [B][Q][k] ascending with -1 padding, n_sel int32 [B][Q],
    mask uint8 [B][Q][N] or None, bits uint32 [B][Q][ceil(N/32)] or None).
    `tile_stats` are the score bounds index_score wrote for these scores.
    `allowed` (uint8 [B][N]) and `allowed_bits` (int32 [B][ceil(N/32)], e.g.
    the gate's fetched set) restrict the eligible entries, and so does
    `n_valid` (int32 [B][Q]: only entries j < n_valid[b][t], the causal
    prefix of a prefill query)."""
    B, Q, N = scores.shape
    dev = scores.device
    ids = torch.empty((B, Q, k), dtype=torch.int32, device=dev) if ids is None else ids
    n_sel = torch.empty((B, Q), dtype=torch.int32, device=dev) if n_sel is None else n_sel
    mask = torch.empty((B, Q, N), dtype=torch.uint8, device=dev) if want_mask else None
    if bits is None and want_bits:
        bits = torch.empty((B, Q, (N + 31) // 32), dtype=torch.int32, device=dev)
    a = topk_args(scores, k, allowed, ids, n_sel, mask, bits, tile_stats=tile_stats, allowed_bits=allowed_bits,
                  n_valid=n_valid)
    if ws is None:
        ws = workspace(workspace_size(OP_TOPK, a), dev)
    _check(lib().lidx_topk_select(C.byref(a), C.c_void_p(ws.data_ptr()), ws.numel(), _stream(stream)),
           "lidx_topk_select")
    return ids, n_sel, mask, bits


def attn_args(q, kv: DeviceKV, N, ids, n_sel, swa: Optional[DeviceKV], swa_len, scale, out, lse,
              flags=0, n_dense=0) -> AttnArgs:
    """ids None with n_dense > 0: the dense rows 0..n_dense-1 (HCA layers)."""
    B, H, D = q.shape
    n_ids = n_dense if ids is None else ids.shape[-1]
    ld_ids = 0 if ids is None else ids.stride(0)
    swa_a = swa.args() if swa is not None else KVArgs(kv.dtype, kv.dim, None, None, None, 0, 0, 0, 0)
    return AttnArgs(B, H, _qdtype(q), q.data_ptr(), kv.args(), N, _ptr(ids), n_ids, ld_ids, _ptr(n_sel),
                    swa_a, swa_len if swa is not None else 0, float(scale), out.data_ptr(), _ptr(lse), flags)


def sparse_attn_decode(q: torch.Tensor, kv: DeviceKV, N: int, ids: torch.Tensor, n_sel: torch.Tensor = None,
                       swa: DeviceKV = None, swa_len: int = 0, scale: float = None, *, out=None, lse=None,
                       want_lse=True, ws=None, stream=None, n_dense=0):
    """MQA decode attention of q [B][H][512] over rows ids [B][n] (-1 skipped;
    the first n_sel[b] when given) of kv plus swa rows 0..swa_len-1.  With
    ids None the rows are 0..n_dense-1 of every sequence, read whole (the HCA
    layers: every compressed entry, no top-k).

    Returns (out float32 [B][H][512], lse float32 [B][H] or None)."""
    B, H, D = q.shape
    if scale is None:
        scale = D ** -0.5
    out = torch.empty((B, H, D), dtype=torch.float32, device=q.device) if out is None else out
    if want_lse and lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    a = attn_args(q, kv, N, ids, n_sel, swa, swa_len, scale, out, lse, n_dense=n_dense)
    if ws is None:
        ws = workspace(workspace_size(OP_ATTN, a), q.device)
    _check(lib().lidx_sparse_attn_decode(C.byref(a), C.c_void_p(ws.data_ptr()), ws.numel(), _stream(stream)),
           "lidx_sparse_attn_decode")
    return out, lse


def decode_args(q_idx, w, keys: DeviceKV, N: int, k: int, q_attn, kv: DeviceKV, swa: Optional[DeviceKV],
                swa_len: int, scale: float, out, lse=None, scores=None, ids=None, n_sel=None, prefetch=(),
                flags=0) -> DecodeArgs:
    """Argument struct of lidx_decode_layer; q_idx [B][H][128] (or [B][1][H][128]),
    w [B][H], q_attn [B][64][512]; `prefetch` is up to two (pointer, bytes)
    pairs pulled into L2 while the layer runs."""
    B = q_attn.shape[0]
    H = w.shape[-1]
    swa_a = swa.args() if swa is not None else KVArgs(kv.dtype, kv.dim, None, None, None, 0, 0, 0, 0)
    pf = list(prefetch)[:2] + [(None, 0)] * (2 - len(list(prefetch)[:2]))
    return DecodeArgs(B, H, N, k, q_idx.data_ptr(), w.data_ptr(), keys.args(), q_attn.shape[1], q_attn.data_ptr(),
                      kv.args(), swa_a, swa_len if swa is not None else 0, float(scale), out.data_ptr(), _ptr(lse),
                      _ptr(scores), 0 if scores is None else scores.stride(-2) if scores.dim() > 1 else N,
                      _ptr(ids), _ptr(n_sel), (C.c_void_p * 2)(*[x[0] for x in pf]),
                      (C.c_uint64 * 2)(*[x[1] for x in pf]), flags)


def decode_layer(q_idx: torch.Tensor, w: torch.Tensor, keys: DeviceKV, N: int, k: int, q_attn: torch.Tensor,
                 kv: DeviceKV, swa: DeviceKV = None, swa_len: int = 0, scale: float = None, *, out=None, lse=None,
                 want_lse=True, scores=None, ids=None, n_sel=None, prefetch=(), flags=0, ws=None, stream=None):
    """One CSA decode layer in one launch: index scores -> top-k -> sparse
    attention over the selected rows plus the window (lidx_decode_layer).
    Returns (out [B][64][512], lse [B][64] or None); `scores`, `ids` and
    `n_sel` are filled when given.  `ws` must be zeroed before its first
    use (workspace() is); the call leaves it ready for the next one."""
    B = q_attn.shape[0]
    if scale is None:
        scale = q_attn.shape[-1] ** -0.5
    out = torch.empty((B, q_attn.shape[1], 512), dtype=torch.float32, device=q_attn.device) if out is None else out
    if want_lse and lse is None:
        lse = torch.empty((B, q_attn.shape[1]), dtype=torch.float32, device=q_attn.device)
    a = decode_args(q_idx, w, keys, N, k, q_attn, kv, swa, swa_len, scale, out, lse, scores, ids, n_sel, prefetch,
                    flags)
    if ws is None:
        ws = workspace(workspace_size(OP_DECODE, a), q_attn.device)
    _check(lib().lidx_decode_layer(C.byref(a), C.c_void_p(ws.data_ptr()), ws.numel(), _stream(stream)),
           "lidx_decode_layer")
    return out, lse


def cache_append(x: torch.Tensor, cache: DeviceKV, pos: torch.Tensor, capacity: int, ring: int = 0, *,
                 ws=None, stream=None, flags=0):
    """Quantise the new rows x [B][R][dim] (float32) into `cache`'s format
    and write row r of sequence b at row pos[b] + r of its region (mod
    `ring` when ring > 0: the sliding window); see lidx_cache_append."""
    B, R, dim = x.shape
    assert x.dtype == torch.float32 and x.is_contiguous() and pos.dtype == torch.int32 and dim == cache.dim
    a = AppendArgs(B, R, x.data_ptr(), cache.args(), capacity, pos.data_ptr(), ring, flags)
    if ws is None:
        ws = workspace(workspace_size(OP_APPEND, a), x.device)
    _check(lib().lidx_cache_append(C.byref(a), C.c_void_p(ws.data_ptr()), ws.numel(), _stream(stream)),
           "lidx_cache_append")
    return ws


def selection_eval(ops: int, *, L=1, T=1, H=1, N, qa=None, kv: DeviceKV = None, scale=None, probs=None,
                   top_p=(3, 5), topp_bits=None, min_votes=3, vote_bits=None, window_bits=None,
                   gate_logits=None, gate_bias=0.0, fetched_bits=None, set_a=None, ld_a=None, set_b=None,
                   ld_b=None, n_pairs=0, counts=None, index_scores=None, ws=None, stream=None):
    """Run the requested evaluation steps (EVAL_* bit mask), in the order
    GOLDEN (or GOLDEN_INDEX: probs as the softmax of index_scores [L*T][>= N]
    rows), TOPP, VOTE, LSA, OVERLAP.  Output tensors must be given by the
    caller (see lidx_eval_args for shapes); returns them in a dict."""
    dev = None
    for t in (qa, probs, topp_bits, gate_logits, set_a, index_scores):
        if t is not None:
            dev = t.device
            break
    kva = kv.args() if kv is not None else KVArgs()
    if scale is None:
        scale = 512 ** -0.5
    a = EvalArgs(ops, L, T, H, N, _qdtype(qa) if qa is not None else BF16, _ptr(qa), kva, float(scale),
                 _ptr(probs), top_p[0], top_p[1], _ptr(topp_bits), min_votes, _ptr(vote_bits), _ptr(window_bits),
                 0 if gate_logits is None else gate_logits.shape[0], _ptr(gate_logits), float(gate_bias),
                 _ptr(fetched_bits), n_pairs, _ptr(set_a),
                 (set_a.stride(0) if set_a is not None and set_a.dim() > 1 else 0) if ld_a is None else ld_a,
                 _ptr(set_b),
                 (set_b.stride(0) if set_b is not None and set_b.dim() > 1 else 0) if ld_b is None else ld_b,
                 _ptr(counts), _ptr(index_scores),
                 0 if index_scores is None else index_scores.stride(-2) if index_scores.dim() > 1 else N)
    if ws is None:
        ws = workspace(workspace_size(OP_EVAL, a), dev)
    _check(lib().lidx_selection_eval(C.byref(a), C.c_void_p(ws.data_ptr()), ws.numel(), _stream(stream)),
           "lidx_selection_eval")
    return dict(probs=probs, topp_bits=topp_bits, vote_bits=vote_bits, window_bits=window_bits,
                fetched_bits=fetched_bits, counts=counts)


def read_device_status(ws: torch.Tensor, stream=None) -> int:
    """Synchronise the stream, return and clear the workspace status word."""
    s = C.c_uint32(0)
    _check(lib().lidx_read_device_status(C.c_void_p(ws.data_ptr()), C.byref(s), _stream(stream)),
           "lidx_read_device_status")
    return s.value


NOALLOC_SCRATCH_BYTES = 16 << 20


def sparse_attn_decode_noalloc(q: torch.Tensor, kv: DeviceKV, N: int, ids: torch.Tensor, n_sel: torch.Tensor = None,
                               swa: DeviceKV = None, swa_len: int = 0, scale: float = None, *, out=None, lse=None,
                               want_lse=True, dev_status: torch.Tensor = None, stream=None):
    """sparse_attn_decode for callers that cannot allocate device memory when
    they call (a plugin hosted by a runtime that offers no scratch allocator,
    a serving loop that forbids cudaMalloc after start-up): the split-K
    scratch lives in a fixed 16 MiB device array owned by the library, shared
    by all calls -- calls that overlap on the GPU race on it.  The first call
    on a device should come before any stream capture.  Requests needing more
    scratch than the array holds raise LidxError(ERR_WORKSPACE).  `out` and
    `lse` are allocated here only when not given."""
    l = lib()
    f = l.lidx_sparse_attn_decode_noalloc
    f.restype = C.c_int
    f.argtypes = [C.POINTER(AttnArgs), C.c_void_p, C.c_void_p]
    B, H, D = q.shape
    if scale is None:
        scale = D ** -0.5
    out = torch.empty((B, H, D), dtype=torch.float32, device=q.device) if out is None else out
    if want_lse and lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    a = attn_args(q, kv, N, ids, n_sel, swa, swa_len, scale, out, lse)
    _check(f(C.byref(a), C.c_void_p(_ptr(dev_status)), _stream(stream)), "lidx_sparse_attn_decode_noalloc")
    return out, lse
