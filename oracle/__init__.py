"""CPU oracle (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product library never uses it.  The
arithmetic lives in ``oracle.c`` (plain C, double precision); this module only
compiles it on first use and marshals numpy arrays into it.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

F32, BF16, E4M3 = 0, 1, 2
_DT = {"f32": F32, "bf16": BF16, "e4m3": E4M3}

ERRORS = {0: "ok", 1: "invalid argument", 2: "nan", 3: "out of range", 4: "no memory"}


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (plain -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=gnu11", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Rows(C.Structure):
    _fields_ = [("dtype", C.c_int32), ("dim", C.c_int32), ("data", C.c_void_p),
                ("scale", C.c_void_p), ("rope", C.c_void_p), ("ld", C.c_int64),
                ("ld_scale", C.c_int64), ("ld_rope", C.c_int64)]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = C.CDLL(build())
            P = C.c_void_p
            I, I64, D = C.c_int, C.c_int64, C.c_double
            RP = C.POINTER(_Rows)
            sig = {
                "orc_decode_bf16": (C.c_double, [C.c_uint16]),
                "orc_decode_e4m3": (C.c_double, [C.c_uint8]),
                "orc_decode_e8m0": (C.c_double, [C.c_uint8]),
                "orc_decode_rows": (I, [RP, I64, P]),
                "orc_encode_e4m3": (C.c_uint8, [C.c_double]),
                "orc_encode_bf16": (C.c_uint16, [C.c_float]),
                "orc_e8m0_for": (C.c_uint8, [C.c_double]),
                "orc_encode_rows": (I, [P, I64, I, I, P, P, P, P]),
                "orc_index_score": (I, [I, I, I, I, RP, P, RP, I64, P, I64, P, P]),
                "orc_topk": (I, [I, I, P, P, P, P, P]),
                "orc_attn": (I, [I, RP, RP, I, P, I, RP, I, D, P, P]),
                "orc_golden": (I, [I, I, I, RP, RP, D, P]),
                "orc_golden_index": (I, [I, I, P, I64, P]),
                "orc_topp": (I, [I, P, C.c_uint32, C.c_uint32, I, P, P]),
                "orc_vote": (I, [I, I, P, I, P]),
                "orc_union": (I, [I, I, P, P]),
                "orc_lsa_gate": (I, [I, I, P, C.c_float, P]),
                "orc_overlap": (I, [I, P, P, P]),
            }
            for name, (res, args) in sig.items():
                f = getattr(lib, name)
                f.restype = res
                f.argtypes = args
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _check(rc):
    if rc != 0:
        raise OracleError(ERRORS.get(rc, str(rc)))


def _rows(kv):
    """synth.KV (or a plain float32 / bf16-bits 2-D array) -> (_Rows, keepalive)."""
    if isinstance(kv, np.ndarray):
        arr = np.ascontiguousarray(kv)
        dt = F32 if arr.dtype == np.float32 else BF16
        if arr.dtype not in (np.float32, np.uint16):
            raise TypeError(arr.dtype)
        arr2 = arr.reshape(-1, arr.shape[-1])
        r = _Rows(dt, arr2.shape[1], arr2.ctypes.data, None, None, arr2.shape[1], 0, 0)
        return r, (arr2,)
    data = np.ascontiguousarray(kv.data)
    keep = [data]
    scale = rope = None
    ld_s = ld_r = 0
    if kv.dtype == "e4m3":
        scale = np.ascontiguousarray(kv.scale)
        rope = np.ascontiguousarray(kv.rope)
        keep += [scale, rope]
        ld_s, ld_r = scale.shape[1], rope.shape[1]
    r = _Rows(_DT[kv.dtype], kv.dim, data.ctypes.data, None if scale is None else scale.ctypes.data,
              None if rope is None else rope.ctypes.data, data.shape[1], ld_s, ld_r)
    return r, tuple(keep)


# ----------------------------------------------------------------- decoders
def decode_bf16(b: int) -> float:
    return _load().orc_decode_bf16(int(b))


def decode_e4m3(b: int) -> float:
    return _load().orc_decode_e4m3(int(b))


def decode_e8m0(b: int) -> float:
    return _load().orc_decode_e8m0(int(b))


def decode_rows(kv) -> np.ndarray:
    """All rows of a KV / array, decoded to float64 [rows][dim]."""
    r, keep = _rows(kv)
    n = keep[0].shape[0]
    out = np.empty((n, r.dim), dtype=np.float64)
    _check(_load().orc_decode_rows(C.byref(r), n, _ptr(out)))
    return out


# ------------------------------------------------------------- the write side
def encode_e4m3(v: float) -> int:
    return int(_load().orc_encode_e4m3(float(v)))


def encode_bf16(x: float) -> int:
    return int(_load().orc_encode_bf16(float(x)))


def e8m0_for(amax: float) -> int:
    return int(_load().orc_e8m0_for(float(amax)))


def encode_rows(x, dtype: str) -> dict:
    """Encode fp32 rows x [rows][dim] for storage (see orc_encode_rows).
    Returns the packed planes: {"data": codes / bf16 bits / fp32,
    "scale": E8M0 codes (e4m3), "rope": bf16 bits (e4m3), "finite": bool}."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    rows, dim = x.shape
    dt = _DT[dtype]
    out = {"scale": None, "rope": None}
    f32 = bits = codes = scales = None
    if dt == F32:
        f32 = np.empty((rows, dim), np.float32)
        out["data"] = f32
    elif dt == BF16:
        bits = np.empty((rows, dim), np.uint16)
        out["data"] = bits
    else:
        codes = np.empty((rows, dim - 64), np.uint8)
        scales = np.empty((rows, (dim - 64) // 64), np.uint8)
        bits = np.empty((rows, 64), np.uint16)
        out.update(data=codes, scale=scales, rope=bits)
    rc = _load().orc_encode_rows(_ptr(x), rows, dim, dt, _ptr(f32), _ptr(bits), _ptr(codes), _ptr(scales))
    if rc not in (0, 2):
        _check(rc)
    out["finite"] = rc == 0
    return out


# ----------------------------------------------------------------- the path
def index_score(q, w, keys, B, Q, H, N, key_batch_rows=None, want_cond=False, want_mag=False):
    """scores float32 [B][Q][N], plus, if requested, float64 [B][Q][N] arrays:
    cond = sum_h |w_h| |q_h . k_j| (the absolute floor of the score tolerance)
    and mag = sum_h |w_h| sum_d |q_hd k_jd| (what a rounding-error bound of
    the sums scales with).  Returns s, (s, cond), (s, mag) or (s, cond, mag).

    q: [B][Q][H][D] (float32 or bf16 bits) or [B][H][D] when Q == 1;
    w: float32 [B][Q][H] / [B][H]; keys: KV with rows b*key_batch_rows + j."""
    qr, qk = _rows(np.asarray(q).reshape(-1, np.asarray(q).shape[-1]))
    kr, kk = _rows(keys)
    w = np.ascontiguousarray(np.asarray(w, dtype=np.float32).reshape(B, Q, H))
    s = np.empty((B, Q, N), dtype=np.float32)
    cond = np.empty((B, Q, N), dtype=np.float64) if want_cond else None
    mag = np.empty((B, Q, N), dtype=np.float64) if want_mag else None
    kbr = N if key_batch_rows is None else key_batch_rows
    _check(_load().orc_index_score(B, Q, H, N, C.byref(qr), _ptr(w), C.byref(kr), kbr,
                                   _ptr(s), N, _ptr(mag), _ptr(cond)))
    out = (s,) + ((cond,) if want_cond else ()) + ((mag,) if want_mag else ())
    return out if len(out) > 1 else s


def topk(scores, k, allowed=None):
    """ids int32 [k] ascending with -1 padding, n_sel, n_nan for one row."""
    s = np.ascontiguousarray(scores, dtype=np.float32).ravel()
    a = None if allowed is None else np.ascontiguousarray(allowed, dtype=np.uint8).ravel()
    ids = np.empty(k, dtype=np.int32)
    n_sel = np.zeros(1, dtype=np.int32)
    n_nan = np.zeros(1, dtype=np.int32)
    _check(_load().orc_topk(s.size, k, _ptr(s), _ptr(a), _ptr(ids), _ptr(n_sel), _ptr(n_nan)))
    return ids, int(n_sel[0]), int(n_nan[0])


def attn(q, kv, N, ids, swa=None, swa_len=0, scale=None, n_ids=None):
    """One decode query: q [H][D]; kv rows [0, N); ids int32; swa rows.
    Returns (out float32 [H][D], lse float32 [H])."""
    qr, qk = _rows(np.asarray(q))
    kr, kk = _rows(kv)
    H = qk[0].shape[0]
    D = kr.dim
    ids = np.ascontiguousarray(ids, dtype=np.int32).ravel()
    n = ids.size if n_ids is None else n_ids
    if swa is not None:
        sr, sk = _rows(swa)
        sp = C.byref(sr)
    else:
        sp, sk = None, ()
    sc = 1.0 / np.sqrt(D) if scale is None else scale
    out = np.empty((H, D), dtype=np.float32)
    lse = np.empty(H, dtype=np.float32)
    _check(_load().orc_attn(H, C.byref(qr), C.byref(kr), N, _ptr(ids), n, sp, swa_len,
                            float(sc), _ptr(out), _ptr(lse)))
    return out, lse


def golden(qa, kv, T, H, N, scale=None):
    """p float32 [T][N] for one layer; qa [T][H][D]."""
    qr, qk = _rows(np.asarray(qa).reshape(-1, np.asarray(qa).shape[-1]))
    kr, kk = _rows(kv)
    sc = 1.0 / np.sqrt(kr.dim) if scale is None else scale
    p = np.empty((T, N), dtype=np.float32)
    _check(_load().orc_golden(T, H, N, C.byref(qr), C.byref(kr), float(sc), _ptr(p)))
    return p


def golden_index(scores):
    """Softmax of each row of scores [..][N] over its N entries (the golden
    probabilities read as a softmax of the indexer logits); float32, same
    shape.  NaN and -inf scores take no mass."""
    s = np.ascontiguousarray(scores, dtype=np.float32)
    N = s.shape[-1]
    R = s.size // N
    p = np.empty(s.shape, dtype=np.float32)
    _check(_load().orc_golden_index(R, N, _ptr(s), N, _ptr(p)))
    return p


TOPP_SHIFT = 40


def topp(p, num=3, den=5, shift=TOPP_SHIFT):
    """(bitset uint32 [ceil(N/32)], count) for one probability row."""
    p = np.ascontiguousarray(p, dtype=np.float32).ravel()
    bits = np.zeros((p.size + 31) // 32, dtype=np.uint32)
    cnt = np.zeros(1, dtype=np.int32)
    _check(_load().orc_topp(p.size, _ptr(p), num, den, shift, _ptr(bits), _ptr(cnt)))
    return bits, int(cnt[0])


def vote(sets, N, min_votes=3):
    sets = np.ascontiguousarray(sets, dtype=np.uint32)
    out = np.zeros((N + 31) // 32, dtype=np.uint32)
    _check(_load().orc_vote(sets.shape[0], N, _ptr(sets), min_votes, _ptr(out)))
    return out


def union(sets, N):
    sets = np.ascontiguousarray(sets, dtype=np.uint32)
    out = np.zeros((N + 31) // 32, dtype=np.uint32)
    _check(_load().orc_union(sets.shape[0], N, _ptr(sets), _ptr(out)))
    return out


def lsa_gate(logits, beta=0.0):
    logits = np.ascontiguousarray(np.atleast_2d(logits), dtype=np.float32)
    G, N = logits.shape
    out = np.zeros((N + 31) // 32, dtype=np.uint32)
    _check(_load().orc_lsa_gate(G, N, _ptr(logits), float(np.float32(beta)), _ptr(out)))
    return out


def overlap(a, b, N):
    a = np.ascontiguousarray(a, dtype=np.uint32)
    b = np.ascontiguousarray(b, dtype=np.uint32)
    c = np.zeros(3, dtype=np.int64)
    _check(_load().orc_overlap(N, _ptr(a), _ptr(b), _ptr(c)))
    return tuple(int(x) for x in c)
