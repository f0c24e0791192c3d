"""Seeded synthetic inputs for the lightning-indexer decode path.

This module is shared by the CPU oracle, the tests and the benchmark.  It only
*produces* input bit patterns (fp32, bf16, OCP E4M3 + E8M0 scale planes); it
holds none of the method's arithmetic (no scoring, selection, softmax or
decoding of the stored formats).

Workload shapes follow the workloads the source pages describe:

* DeepSeek-V4-Flash architecture post (Part 6), section (A): CSA layers keep
  4:1-compressed entries whose attention rows (``attn_comp_kv``) are 512 wide;
  section (B): the lightning indexer scores them with its own 128-d index keys
  (``index_comp_kv``) and keeps the top-512 (1024 for the Pro variant), plus a
  128-token sliding window; "why you cannot quantise the KV": non-RoPE dims are
  FP8 E4M3 with one power-of-two scale per 64 elements, RoPE dims bf16.
* FlashMemory-DeepSeek-V4 write-up, sections 2.2 and 4.1: a gate every
  tau=64 steps at layers 10/12/20 combined by OR.

Every tensor draws from its own numpy ``SeedSequence`` keyed by
(seed, tensor tag, layer, batch), so any slice can be regenerated alone.
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import math
import os
from typing import Optional

import numpy as np

# ----------------------------------------------------------------------------
# tensor tags (substream keys)
# ----------------------------------------------------------------------------
TAG_Q_IDX = 1
TAG_W = 2
TAG_KEYS = 3
TAG_KV = 4
TAG_SWA = 5
TAG_Q_ATTN = 6
TAG_PLANT = 7
TAG_GATE_Q = 8
TAG_GATE_U = 9
TAG_SCORES = 10
TAG_PROBS = 11
TAG_BITS = 12
TAG_IDS = 13


def rng(seed: int, tag: int, layer: int = 0, b: int = 0) -> np.random.Generator:
    """Independent PCG64 substream for one tensor slice."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tag, layer, b])))


# ----------------------------------------------------------------------------
# storage encoders (input production only)
# ----------------------------------------------------------------------------
def bf16_bits(x) -> np.ndarray:
    """float64/float32 array -> bf16 bit patterns (uint16), round-to-nearest-even
    via float32.  NaN stays NaN."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    nan = np.isnan(f)
    out = rounded.astype(np.uint16)
    out[nan] = 0x7FC0
    return out


def bf16_value(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 values (bit placement, used to build
    derived inputs such as the planted direction)."""
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32)


_E4M3_MAX = 448.0


def e4m3_bits(v: np.ndarray) -> np.ndarray:
    """Encode float64 values (already divided by their block scale) as OCP
    E4M3FN bytes: bias 7, 3 mantissa bits, subnormals below 2^-6, largest
    finite 448, no infinities; round-to-nearest-even, saturating to +-448."""
    v = np.asarray(v, dtype=np.float64)
    sign = (v < 0) | ((v == 0) & np.signbit(v))
    a = np.minimum(np.abs(v), _E4M3_MAX)
    # exponent of the binade (subnormal range shares the 2^-6 binade quantum)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -6.0)
    quantum = np.exp2(e - 3.0)
    q = np.round(a / quantum) * quantum          # numpy rounds half to even
    q = np.minimum(q, _E4M3_MAX)
    with np.errstate(divide="ignore"):
        e2 = np.floor(np.log2(np.where(q > 0, q, 1.0)))
    normal = q >= 2.0 ** -6
    exp_field = np.where(normal, e2 + 7.0, 0.0)
    mant = np.where(normal, q / np.exp2(e2) * 8.0 - 8.0, q / 2.0 ** -9)
    code = (exp_field.astype(np.int64) << 3) | np.rint(mant).astype(np.int64)
    code = code | (sign.astype(np.int64) << 7)
    return code.astype(np.uint8)


def e4m3_quantize_rows(x: np.ndarray, block: int = 64):
    """Quantise rows ``x[..., n*block]`` (float64) into E4M3 bytes plus one E8M0
    scale byte per block: scale exponent ``e = ceil(log2(amax/448))`` so the
    block's largest magnitude lands at or below 448; code ``e + 127``."""
    x = np.asarray(x, dtype=np.float64)
    nblk = x.shape[-1] // block
    xb = x.reshape(x.shape[:-1] + (nblk, block))
    amax = np.max(np.abs(xb), axis=-1)
    with np.errstate(divide="ignore"):
        e = np.ceil(np.log2(np.where(amax > 0, amax / _E4M3_MAX, 1.0)))
    e = np.clip(e, -127, 127)
    codes = e4m3_bits(xb / np.exp2(e)[..., None]).reshape(x.shape)
    scale = (e + 127).astype(np.uint8)
    return codes, scale


# ----------------------------------------------------------------------------
# KV planes
# ----------------------------------------------------------------------------
@dataclasses.dataclass
class KV:
    """Host-side rows in one of the three storage formats.

    dtype "f32":  data float32 [rows][dim]
    dtype "bf16": data uint16  [rows][dim] (bf16 bits)
    dtype "e4m3": data uint8 [rows][dim-64] E4M3 codes, scale uint8
                  [rows][(dim-64)/64] E8M0 codes, rope uint16 [rows][64] bf16;
                  logical row = [dequantised non-RoPE dims | RoPE dims].
    """
    dtype: str
    dim: int
    data: np.ndarray
    scale: Optional[np.ndarray] = None
    rope: Optional[np.ndarray] = None

    @property
    def rows(self) -> int:
        return self.data.shape[0]

    def slice(self, r0: int, r1: int) -> "KV":
        return KV(self.dtype, self.dim, self.data[r0:r1],
                  None if self.scale is None else self.scale[r0:r1],
                  None if self.rope is None else self.rope[r0:r1])

    def nbytes(self) -> int:
        n = self.data.nbytes
        if self.scale is not None:
            n += self.scale.nbytes
        if self.rope is not None:
            n += self.rope.nbytes
        return n


def encode_rows(x64: np.ndarray, dtype: str) -> KV:
    """Store float64 rows [rows][dim] in the requested format."""
    rows, dim = x64.shape
    if dtype == "f32":
        return KV("f32", dim, np.ascontiguousarray(x64.astype(np.float32)))
    if dtype == "bf16":
        return KV("bf16", dim, bf16_bits(x64))
    if dtype == "e4m3":
        codes, scale = e4m3_quantize_rows(x64[:, : dim - 64])
        return KV("e4m3", dim, np.ascontiguousarray(codes), np.ascontiguousarray(scale),
                  bf16_bits(x64[:, dim - 64:]))
    raise ValueError(dtype)


def concat_kv(parts) -> KV:
    p0 = parts[0]
    return KV(p0.dtype, p0.dim, np.concatenate([p.data for p in parts]),
              None if p0.scale is None else np.concatenate([p.scale for p in parts]),
              None if p0.rope is None else np.concatenate([p.rope for p in parts]))


# ----------------------------------------------------------------------------
# workload specs
# ----------------------------------------------------------------------------
@dataclasses.dataclass
class DecodeSpec:
    """One decode workload: ``layers`` independent CSA layers, each with a batch
    of ``B`` sequences of ``N`` compressed entries."""
    name: str
    seed: int
    B: int
    N: int
    H: int            # index heads == attention query heads
    k: int
    layers: int = 1
    key_dtype: str = "bf16"     # f32 | bf16 | e4m3
    q_dtype: str = "bf16"       # f32 | bf16 (index and attention queries)
    kv_dtype: str = "bf16"      # storage of comp_kv and SWA rows
    swa: int = 128
    plant: bool = False
    D_idx: int = 128
    D_attn: int = 512

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D_attn)


# The workloads: a tiny fp32 parity case, one 64K decode token over 21 CSA
# layers, a planted 128K batch of 32, and the 500K Pro batch of 4 in FP8.
TINY_1K_F32 = DecodeSpec("tiny-1k-f32", seed=0, B=1, N=1024, H=16, k=64, key_dtype="f32",
                         q_dtype="f32", kv_dtype="f32")
DECODE_64K = DecodeSpec("decode-64k-b1-x21", seed=1, B=1, N=16384, H=64, k=512, layers=21)
DECODE_128K_B32 = DecodeSpec("decode-128k-b32-planted", seed=2, B=32, N=32768, H=64, k=512, plant=True)
DECODE_500K_FP8 = DecodeSpec("decode-500k-b4-pro-fp8", seed=3, B=4, N=125000, H=64, k=1024,
                             key_dtype="e4m3", kv_dtype="e4m3")


@dataclasses.dataclass
class EvalSpec:
    """tau-window selection evaluation: ``L`` CSA layers, ``T`` queries that all
    see the same ``N`` entries, gate at the CSA stack indices of model layers
    10/12/20."""
    name: str = "eval-window-64x21-32k"
    seed: int = 4
    L: int = 21
    T: int = 64
    H: int = 64
    N: int = 32768
    k: int = 512
    D_idx: int = 128
    D_attn: int = 512
    gate_layers: tuple = (4, 5, 9)
    gate_heads: int = 64
    top_p_num: int = 3
    top_p_den: int = 5
    min_votes: int = 3

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D_attn)


EVAL_WINDOW = EvalSpec()


def scaled(spec, **kw):
    return dataclasses.replace(spec, **kw)


# ----------------------------------------------------------------------------
# decode inputs
# ----------------------------------------------------------------------------
def _normal(g: np.random.Generator, shape, sd: float) -> np.ndarray:
    return g.standard_normal(shape) * sd


def decode_layer(spec: DecodeSpec, layer: int = 0) -> dict:
    """Inputs of one CSA layer of a decode workload.

    Returns a dict with
      q_idx  [B][H][128]   index queries  ~ N(0,1)/sqrt(128)  (spec.q_dtype)
      w      [B][H]        head weights   ~ U(0,1)            float32
      keys   KV rows B*N, dim 128, ~ N(0,1)/sqrt(128)
      kv     KV rows B*N, dim 512, ~ N(0,1)
      swa    KV rows B*swa, dim 512, ~ N(0,1)
      q_attn [B][H][512]   attention queries ~ N(0,1)
      planted int32 [B][k] (only when spec.plant)
    """
    B, N, H = spec.B, spec.N, spec.H
    s, l = spec.seed, layer
    sd_idx = 1.0 / math.sqrt(spec.D_idx)

    def one(b):  # every array of sequence b comes from its own streams
        q = _normal(rng(s, TAG_Q_IDX, l, b), (H, spec.D_idx), sd_idx)
        w = rng(s, TAG_W, l, b).random(H).astype(np.float32)
        k = _normal(rng(s, TAG_KEYS, l, b), (N, spec.D_idx), sd_idx)
        q_st = q.astype(np.float32) if spec.q_dtype == "f32" else bf16_bits(q)
        rows = None
        if spec.plant:
            # planted rows: shift chosen rows along g = sum_h q_h / |sum_h q_h|
            # so the head-mean of q_h . k rises by 3 sigma (sigma = 1/sqrt(128)).
            qv = q_st.astype(np.float64) if spec.q_dtype == "f32" else bf16_value(q_st).astype(np.float64)
            gsum = qv.sum(axis=0)
            gnorm = np.linalg.norm(gsum)
            ghat = gsum / gnorm
            c = 3.0 * sd_idx * H / gnorm
            rows = np.sort(rng(s, TAG_PLANT, l, b).choice(N, size=spec.k, replace=False))
            k[rows] += c * ghat
            rows = rows.astype(np.int32)
        key = encode_rows(k, spec.key_dtype)
        x = _normal(rng(s, TAG_KV, l, b), (N, spec.D_attn), 1.0)
        kv = encode_rows(x, spec.kv_dtype)
        sw = _normal(rng(s, TAG_SWA, l, b), (spec.swa, spec.D_attn), 1.0)
        swa = encode_rows(sw, spec.kv_dtype)
        qa = _normal(rng(s, TAG_Q_ATTN, l, b), (H, spec.D_attn), 1.0)
        qa = qa.astype(np.float32) if spec.q_dtype == "f32" else bf16_bits(qa)
        return q_st, w, key, kv, swa, qa, rows

    if B > 1 and B * N >= 1 << 16:
        with concurrent.futures.ThreadPoolExecutor(min(B, os.cpu_count() or 1)) as ex:
            parts = list(ex.map(one, range(B)))
    else:
        parts = [one(b) for b in range(B)]
    qs, ws, keys, kvs, swas, qas, planted = (list(t) for t in zip(*parts))
    out = dict(q_idx=np.stack(qs), w=np.stack(ws), keys=concat_kv(keys), kv=concat_kv(kvs),
               swa=concat_kv(swas), q_attn=np.stack(qas))
    if spec.plant:
        out["planted"] = np.stack(planted)
    return out


def model_layer(spec: DecodeSpec, layer: int) -> dict:
    """Inputs of model layer `layer` of the hybrid schedule for one decode
    token (architecture post, section (A): layers 0-1 sliding window only,
    even layers 2-42 CSA, odd layers 3-41 HCA).  A CSA layer is
    decode_layer(spec, (layer - 2) // 2); an HCA layer has spec.N // 32
    compressed rows (128:1 against CSA's 4:1) of width 512 ~ N(0,1), its
    window and attention queries; an SWA layer has its window and queries.
    Returns a dict with "kind" and the arrays."""
    if layer >= 2 and layer % 2 == 0:
        return dict(kind="csa", **decode_layer(spec, (layer - 2) // 2))
    sub = dataclasses.replace(spec, N=max(1, spec.N // 32), plant=False)
    x = decode_layer(sub, 1000 + layer)  # its own streams: layer ids 1000+ are not used by CSA layers
    if layer < 2:
        return dict(kind="swa", swa=x["swa"], q_attn=x["q_attn"])
    return dict(kind="hca", N=sub.N, kv=x["kv"], swa=x["swa"], q_attn=x["q_attn"])


# ----------------------------------------------------------------------------
# selection-eval inputs
# ----------------------------------------------------------------------------
def eval_layer(spec: EvalSpec, layer: int) -> dict:
    """Inputs of one layer of the tau-window evaluation.

      q_idx [T][H][128] bf16, w [T][H] U(0,1), keys [N][128] bf16,
      qa [T][H][512] bf16 ~ N(0,1), kv [N][512] bf16 ~ N(0,1)
    """
    s, l = spec.seed, layer
    sd_idx = 1.0 / math.sqrt(spec.D_idx)
    q = bf16_bits(_normal(rng(s, TAG_Q_IDX, l), (spec.T, spec.H, spec.D_idx), sd_idx))
    w = rng(s, TAG_W, l).random((spec.T, spec.H)).astype(np.float32)
    keys = encode_rows(_normal(rng(s, TAG_KEYS, l), (spec.N, spec.D_idx), sd_idx), "bf16")
    qa = bf16_bits(_normal(rng(s, TAG_Q_ATTN, l), (spec.T, spec.H, spec.D_attn), 1.0))
    kv = encode_rows(_normal(rng(s, TAG_KV, l), (spec.N, spec.D_attn), 1.0), "bf16")
    return dict(q_idx=q, w=w, keys=keys, qa=qa, kv=kv)


def eval_gate(spec: EvalSpec) -> dict:
    """Memory-indexer gate inputs for one tau-window: per gate layer one query
    g [Hg][128] bf16 ~ N(0,1)/sqrt(128) and signed head weights u [Hg] ~ U(-1,1)
    (trained gate weights can be negative), bias beta = 0."""
    sd_idx = 1.0 / math.sqrt(spec.D_idx)
    g = np.stack([bf16_bits(_normal(rng(spec.seed, TAG_GATE_Q, l), (spec.gate_heads, spec.D_idx), sd_idx))
                  for l in spec.gate_layers])
    u = np.stack([(rng(spec.seed, TAG_GATE_U, l).random(spec.gate_heads) * 2.0 - 1.0).astype(np.float32)
                  for l in spec.gate_layers])
    return dict(g=g, u=u, beta=np.float32(0.0))


# ----------------------------------------------------------------------------
# raw arrays for the selection and set kernels
# ----------------------------------------------------------------------------
def random_scores(seed: int, rows: int, N: int, kind: str = "normal") -> np.ndarray:
    """fp32 score rows for selection tests.

    kind "normal": N(1,0.25) like the ReLU-head sums; "ties": small integers so
    many entries tie exactly; "signed": N(0,1) with +-0.0 and denormals mixed in;
    "const": all equal.
    """
    g = rng(seed, TAG_SCORES, rows, N)
    if kind == "normal":
        return (1.0 + 0.25 * g.standard_normal((rows, N))).astype(np.float32)
    if kind == "ties":
        return g.integers(0, 16, size=(rows, N)).astype(np.float32)
    if kind == "signed":
        x = g.standard_normal((rows, N)).astype(np.float32)
        m = g.random((rows, N))
        x[m < 0.05] = 0.0
        x[(m >= 0.05) & (m < 0.1)] = -0.0
        x[(m >= 0.1) & (m < 0.12)] = np.float32(1e-40)
        x[(m >= 0.12) & (m < 0.14)] = np.float32(-1e-40)
        return x
    if kind == "const":
        return np.full((rows, N), 0.5, dtype=np.float32)
    raise ValueError(kind)


def random_probs(seed: int, rows: int, N: int, concentration: float = 1.0) -> np.ndarray:
    """fp32 probability rows (each sums to ~1) with a heavy-ish head:
    softmax of N(0, concentration^2) logits, with some exact duplicates."""
    g = rng(seed, TAG_PROBS, rows, N)
    z = g.standard_normal((rows, N)) * concentration
    z[:, 1::7] = z[:, 0:1]  # exact duplicates -> ties
    e = np.exp(z - z.max(axis=1, keepdims=True))
    return (e / e.sum(axis=1, keepdims=True)).astype(np.float32)


def random_bits(seed: int, rows: int, N: int, density: float) -> np.ndarray:
    """uint32 bitsets [rows][ceil(N/32)] with zero padding beyond N."""
    g = rng(seed, TAG_BITS, rows, N)
    dense = g.random((rows, N)) < density
    return pack_bits(dense)


def pack_bits(dense: np.ndarray) -> np.ndarray:
    """bool [rows][N] -> uint32 [rows][ceil(N/32)], bit j%32 of word j/32."""
    dense = np.atleast_2d(dense)
    rows, N = dense.shape
    W = (N + 31) // 32
    pad = np.zeros((rows, W * 32), dtype=np.uint8)
    pad[:, :N] = dense
    b = pad.reshape(rows, W, 32).astype(np.uint64) << np.arange(32, dtype=np.uint64)
    return b.sum(axis=2).astype(np.uint32)


def unpack_bits(bits: np.ndarray, N: int) -> np.ndarray:
    bits = np.atleast_2d(bits)
    w = bits[:, :, None].astype(np.uint64) >> np.arange(32, dtype=np.uint64)
    return (w & 1).astype(bool).reshape(bits.shape[0], -1)[:, :N]
