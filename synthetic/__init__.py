"""Seeded synthetic inputs for the routed, block-quantized MoE FFN layer.

This module is shared by the CUDA path's tests/bench and by the oracle's tests.
It only *produces inputs*: random activations, router weights and biases,
routing traces, and ggml-style block encodings (Q8_0 / Q4_0) of random expert
weights.  It holds none of the layer's arithmetic (no dequantization, routing,
softmax, SwiGLU or combine); the decoders live separately in ``oracle/`` and in
the CUDA library and share no code.

Block formats (the quant types named in the FreeToken fork README, "Quant
types" table: the Standard family Q4_0, Q4_1, Q5_0, Q5_1, Q8_0; the byte
layouts are ggml's published ones), 32 weights per block, blocks run along the
reduction dimension of each weight row, all fields little endian:

* Q8_0: ``{fp16 d; int8 qs[32]}``  (34 bytes), value ``qs[i] * d``.
* Q4_0: ``{fp16 d; uint8 qs[16]}`` (18 bytes), value ``(q_i - 8) * d`` where
  byte ``j`` holds element ``j`` in its low nibble and element ``j + 16`` in its
  high nibble (the GGUF order).
* Q4_1: ``{fp16 d; fp16 m; uint8 qs[16]}`` (20 bytes), value ``q_i * d + m``.
* Q5_0: ``{fp16 d; uint8 qh[4]; uint8 qs[16]}`` (22 bytes), value
  ``(q_i - 16) * d``; bit ``i`` of the 32-bit word ``qh`` is bit 4 of ``q_i``,
  ``qs`` holds the low four bits as in Q4_0.
* Q5_1: ``{fp16 d; fp16 m; uint8 qh[4]; uint8 qs[16]}`` (24 bytes), value
  ``q_i * d + m``.

K-quants (same table, K-quants row; ggml's published layouts), 256 weights
per block:

* Q4_K: ``{fp16 d; fp16 dmin; uint8 scales[12]; uint8 qs[128]}`` (144 bytes):
  eight 32-weight sub-blocks with 6-bit scales ``sc_j`` and mins ``m_j``
  (``j < 4``: low six bits of ``scales[j]`` / ``scales[j+4]``; ``j >= 4``:
  low / high nibble of ``scales[j+4]`` plus the top two bits of
  ``scales[j-4]`` / ``scales[j]``); value ``d * sc_j * q - dmin * m_j``;
  weight ``64c + l`` is the low nibble of ``qs[32c + l]``, weight
  ``64c + 32 + l`` its high nibble.
* Q6_K: ``{uint8 ql[128]; uint8 qh[64]; int8 scales[16]; fp16 d}`` (210
  bytes): value ``d * scales[i // 16] * (q_i - 32)``; weight
  ``128h + 32r + l`` keeps its low four bits in nibble ``r // 2`` of
  ``ql[64h + 32(r % 2) + l]`` and its high two in bits ``2r, 2r+1`` of
  ``qh[32h + l]``.

Expert pools follow the FreeToken fork README, "Known limits": experts stored
back to back as ``expert * nrows * (ncols / 32)`` blocks with no padding and
one quant type for the whole pool.  Per expert, ``W_gate`` and ``W_up`` are
``[F rows][D/32 blocks]`` and ``W_down`` is ``[D rows][F/32 blocks]``.

Workload recipes (shapes, distributions, seeds) are in ``CONFIGS``.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

QK = 32
Q4_0 = "q4_0"
Q4_1 = "q4_1"
Q5_0 = "q5_0"
Q5_1 = "q5_1"
Q8_0 = "q8_0"
Q4_K = "q4_k"
Q6_K = "q6_k"
QTYPES = (Q4_0, Q4_1, Q5_0, Q5_1, Q8_0, Q4_K, Q6_K)
QK_K = 256
# bytes per block and weights per block; a test checks these against
# include/moe.h
BLOCK_BYTES = {Q4_0: 18, Q4_1: 20, Q5_0: 22, Q5_1: 24, Q8_0: 34, Q4_K: 144, Q6_K: 210}
BLOCK_WEIGHTS = {q: (QK_K if q in (Q4_K, Q6_K) else QK) for q in QTYPES}
# ggml type ids, also exported by the C header
GGML_TYPE_ID = {Q4_0: 2, Q4_1: 3, Q5_0: 6, Q5_1: 7, Q8_0: 8, Q4_K: 12, Q6_K: 14}


def row_bytes(ncols: int, qtype: str) -> int:
    """Bytes of one weight row of ncols weights (a multiple of the block)."""
    assert ncols % BLOCK_WEIGHTS[qtype] == 0
    return ncols // BLOCK_WEIGHTS[qtype] * BLOCK_BYTES[qtype]


# --------------------------------------------------------------------------
# configurations
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int
    D: int
    E: int
    k: int
    F: int
    qtype: str
    x_dtype: str            # "f32" or "bf16"
    y_dtype: str            # "f32" or "bf16"
    router_std: float = 0.02
    expert_std: float = 0.02
    zipf_s: float | None = None          # per-expert router bias (prefill config)
    logits_from_trace: bool = False      # routing logits given directly
    shared_F: int = 0                    # always-on shared expert
    shared_qtype: str = Q8_0             # its block type
    seed: int = 1000
    renorm: bool = True
    T_values: tuple = field(default_factory=tuple)   # documentation only


CONFIGS = {
    # Tiny routed layer: fp32 activations, Q8_0 experts, fp32 output.
    "tiny": LayerConfig("tiny", T=4, D=256, E=8, k=2, F=512, qtype=Q8_0,
                        x_dtype="f32", y_dtype="f32", router_std=0.05,
                        seed=1000),
    # Decode, 30B-A3B-shaped layer in Q4_0 at T in {1, 4, 16}.
    "decode": LayerConfig("decode", T=16, D=2048, E=128, k=8, F=768,
                          qtype=Q4_0, x_dtype="bf16", y_dtype="bf16",
                          seed=1001, T_values=(1, 4, 16)),
    # Prefill, same shapes in Q8_0, T=8192, Zipf(1.1) router bias.
    "prefill": LayerConfig("prefill", T=8192, D=2048, E=128, k=8, F=768,
                           qtype=Q8_0, x_dtype="bf16", y_dtype="bf16",
                           zipf_s=1.1, seed=1002),
    # Wide-expert layer: E=512, top-10, F=512, Q4_0 routed + Q8_0 shared
    # expert, routing logits from a temporal-locality trace, T in {1, 2048}.
    "wide": LayerConfig("wide", T=2048, D=2048, E=512, k=10, F=512,
                        qtype=Q4_0, x_dtype="bf16", y_dtype="bf16",
                        logits_from_trace=True, shared_F=512, seed=1003,
                        T_values=(1, 2048)),
    # Expert-cache streaming: 40 layers of the decode layer in Q8_0.
    "cache": LayerConfig("cache", T=1, D=2048, E=128, k=8, F=768, qtype=Q8_0,
                         x_dtype="bf16", y_dtype="bf16",
                         logits_from_trace=True, seed=1004),
}
CACHE_LAYERS = 40
CACHE_STEPS = 256
CACHE_FRACTION = 0.4


def with_T(cfg: LayerConfig, T: int) -> LayerConfig:
    d = dict(cfg.__dict__)
    d["T"] = T
    return LayerConfig(**d)


def expert_bytes(D: int, F: int, qtype: str) -> tuple[int, int, int]:
    """Bytes of (gate, up, down) of one expert in the pool layout."""
    return F * row_bytes(D, qtype), F * row_bytes(D, qtype), D * row_bytes(F, qtype)


# --------------------------------------------------------------------------
# scalar encodings
# --------------------------------------------------------------------------
def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounding = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _round_half_away(v: np.ndarray) -> np.ndarray:
    return np.sign(v) * np.floor(np.abs(v) + np.float32(0.5))


# --------------------------------------------------------------------------
# block encoders (input generation only)
# --------------------------------------------------------------------------
def quantize_q8_0(w: np.ndarray) -> np.ndarray:
    """Encode rows of float32 weights as Q8_0 blocks.

    ``w``: [rows, cols] with cols % 32 == 0.  Returns uint8 [rows, cols/32*34].
    Scale d = max|w| / 127 per block (fp32), q = round-half-away(w / d),
    d stored as fp16.  An all-zero block gets d = 0, q = 0.
    """
    rows, cols = w.shape
    assert cols % QK == 0
    b = np.ascontiguousarray(w, dtype=np.float32).reshape(rows, cols // QK, QK)
    amax = np.abs(b).max(axis=2)
    d = (amax / np.float32(127.0)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = _round_half_away(b / d[..., None])
    q = np.where(d[..., None] > 0, q, 0)
    q = np.clip(q, -127, 127).astype(np.int8)
    out = np.empty((rows, cols // QK, 34), dtype=np.uint8)
    out[..., 0:2] = d.astype(np.float16).view(np.uint8).reshape(rows, cols // QK, 2)
    out[..., 2:] = q.view(np.uint8)
    return out.reshape(rows, -1)


def quantize_q4_0(w: np.ndarray) -> np.ndarray:
    """Encode rows of float32 weights as Q4_0 blocks.

    Per block: m = the signed weight of largest magnitude (the positive one
    when a positive and a negative weight tie in magnitude), d = -m / 8 so
    that m lands exactly on code 0, q = clamp(round-half-away(w / d) + 8, 0,
    15), d stored as fp16; value (q - 8) * d.  An all-zero block gets d = 0
    and q = 8.  Returns uint8 [rows, cols/32*18].
    """
    rows, cols = w.shape
    assert cols % QK == 0
    b = np.ascontiguousarray(w, dtype=np.float32).reshape(rows, cols // QK, QK)
    hi = b.max(axis=2)
    lo = b.min(axis=2)
    m = np.where(hi >= -lo, hi, lo)
    d = (m / np.float32(-8.0)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = _round_half_away(b / d[..., None]) + 8
    q = np.where(d[..., None] != 0, q, 8)
    q = np.clip(q, 0, 15).astype(np.uint8)
    out = np.empty((rows, cols // QK, 18), dtype=np.uint8)
    out[..., 0:2] = d.astype(np.float16).view(np.uint8).reshape(rows, cols // QK, 2)
    out[..., 2:] = q[..., :16] | (q[..., 16:] << 4)
    return out.reshape(rows, -1)


def _nibble_bytes(q: np.ndarray) -> np.ndarray:
    """Low four bits of codes [..., 32] as 16 bytes: element j low, j+16 high."""
    return (q[..., :16] & 0xF) | ((q[..., 16:] & 0xF) << 4)


def _high_bit_word(q: np.ndarray) -> np.ndarray:
    """Bit 4 of codes [..., 32] as a little-endian 32-bit word (4 bytes)."""
    bits = ((q.astype(np.uint32) >> 4) & 1) << np.arange(QK, dtype=np.uint32)
    w = bits.sum(axis=-1, dtype=np.uint64).astype(np.uint32)
    return np.stack([(w >> (8 * i)) & 0xFF for i in range(4)], axis=-1).astype(np.uint8)


def _f16_bytes(v: np.ndarray) -> np.ndarray:
    """fp16 little-endian bytes [..., 2] of float32 values [...]."""
    h = v.astype(np.float16).view(np.uint16)
    return np.stack([h & 0xFF, h >> 8], axis=-1).astype(np.uint8)


def quantize_min_scale(w: np.ndarray, bits: int) -> np.ndarray:
    """Encode rows of float32 weights as Q4_1 (bits=4) or Q5_1 (bits=5).

    Per block: m = min, d = (max - min) / (2^bits - 1) (fp32), q =
    clamp(floor((w - m) / d + 0.5), 0, 2^bits - 1); d and m stored as fp16;
    value q * d + m.  A constant block gets d = 0 and q = 0.
    """
    rows, cols = w.shape
    assert cols % QK == 0 and bits in (4, 5)
    top = (1 << bits) - 1
    b = np.ascontiguousarray(w, dtype=np.float32).reshape(rows, cols // QK, QK)
    lo = b.min(axis=2)
    d = ((b.max(axis=2) - lo) / np.float32(top)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.floor((b - lo[..., None]) / d[..., None] + np.float32(0.5))
    q = np.where(d[..., None] > 0, q, 0)
    q = np.clip(q, 0, top).astype(np.uint8)
    parts = [_f16_bytes(d), _f16_bytes(lo)]
    if bits == 5:
        parts.append(_high_bit_word(q))
    parts.append(_nibble_bytes(q))
    return np.concatenate(parts, axis=2).reshape(rows, -1)


def quantize_q5_0(w: np.ndarray) -> np.ndarray:
    """Encode rows of float32 weights as Q5_0 blocks.

    As Q4_0 with 32 levels: m = the signed weight of largest magnitude (the
    positive one on a tie), d = -m / 16, q = clamp(round-half-away(w / d) +
    16, 0, 31), d stored as fp16; value (q - 16) * d.  An all-zero block gets
    d = 0 and q = 16.  Returns uint8 [rows, cols/32*22].
    """
    rows, cols = w.shape
    assert cols % QK == 0
    b = np.ascontiguousarray(w, dtype=np.float32).reshape(rows, cols // QK, QK)
    hi = b.max(axis=2)
    lo = b.min(axis=2)
    m = np.where(hi >= -lo, hi, lo)
    d = (m / np.float32(-16.0)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = _round_half_away(b / d[..., None]) + 16
    q = np.where(d[..., None] != 0, q, 16)
    q = np.clip(q, 0, 31).astype(np.uint8)
    return np.concatenate([_f16_bytes(d), _high_bit_word(q), _nibble_bytes(q)],
                          axis=2).reshape(rows, -1)


def quantize_q4_k(w: np.ndarray) -> np.ndarray:
    """Encode rows of float32 weights as Q4_K super-blocks.

    Per 32-weight sub-block j: lo_j = min(min w, 0), s_j = (max w - lo_j) / 15.
    Per super-block: d = max_j s_j / 63, dmin = max_j (-lo_j) / 63 (stored
    fp16); sc_j = clamp(round-half-away(s_j / d), 0, 63), m_j =
    clamp(round-half-away(-lo_j / dmin), 0, 63); q = clamp(floor((w + dmin
    m_j) / (d sc_j) + 1/2), 0, 15) with the stored d, dmin (q = 0 where d sc_j
    is 0).  Returns uint8 [rows, cols/256*144].
    """
    rows, cols = w.shape
    assert cols % QK_K == 0
    nsb = cols // QK_K
    b = np.ascontiguousarray(w, dtype=np.float32).reshape(rows, nsb, 8, 32)
    lo = np.minimum(b.min(axis=3), 0)
    s = ((b.max(axis=3) - lo) / np.float32(15)).astype(np.float32)
    d16 = (s.max(axis=2) / np.float32(63)).astype(np.float16)
    m16 = ((-lo).max(axis=2) / np.float32(63)).astype(np.float16)
    d32, m32 = d16.astype(np.float32), m16.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        sc = np.where(d32[..., None] > 0, _round_half_away(s / d32[..., None]), 0)
        mn = np.where(m32[..., None] > 0, _round_half_away(-lo / m32[..., None]), 0)
    sc = np.clip(sc, 0, 63).astype(np.uint8)
    mn = np.clip(mn, 0, 63).astype(np.uint8)
    eff = d32[..., None] * sc.astype(np.float32)
    off = m32[..., None] * mn.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.floor((b + off[..., None]) / eff[..., None] + np.float32(0.5))
    q = np.where(eff[..., None] > 0, q, 0)
    q = np.clip(q, 0, 15).astype(np.uint8)                         # [rows, nsb, 8, 32]
    s12 = np.zeros((rows, nsb, 12), np.uint8)
    s12[..., 0:4] = (sc[..., 0:4] & 63) | ((sc[..., 4:8] >> 4) << 6)
    s12[..., 4:8] = (mn[..., 0:4] & 63) | ((mn[..., 4:8] >> 4) << 6)
    s12[..., 8:12] = (sc[..., 4:8] & 15) | ((mn[..., 4:8] & 15) << 4)
    qs = (q[..., 0::2, :] | (q[..., 1::2, :] << 4)).reshape(rows, nsb, 128)
    return np.concatenate([_f16_bytes(d32), _f16_bytes(m32), s12, qs], axis=2).reshape(rows, -1)


def quantize_q6_k(w: np.ndarray) -> np.ndarray:
    """Encode rows of float32 weights as Q6_K super-blocks.

    Per 16-weight sub-block j: m_j = the signed weight of largest magnitude
    (the positive one on a tie), s_j = -m_j / 32.  Per super-block: d =
    max_j |s_j| / 127 (stored fp16), sc_j = clamp(round-half-away(s_j / d),
    -128, 127); q = clamp(round-half-away(w / (d sc_j)) + 32, 0, 63) (32 where
    d sc_j is 0).  Returns uint8 [rows, cols/256*210].
    """
    rows, cols = w.shape
    assert cols % QK_K == 0
    nsb = cols // QK_K
    b = np.ascontiguousarray(w, dtype=np.float32).reshape(rows, nsb, 16, 16)
    hi, lo = b.max(axis=3), b.min(axis=3)
    m = np.where(hi >= -lo, hi, lo)
    s = (m / np.float32(-32)).astype(np.float32)
    d16 = (np.abs(s).max(axis=2) / np.float32(127)).astype(np.float16)
    d32 = d16.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        sc = np.where(d32[..., None] > 0, _round_half_away(s / d32[..., None]), 0)
    sc = np.clip(sc, -128, 127).astype(np.int8)
    eff = d32[..., None] * sc.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = _round_half_away(b / eff[..., None]) + 32
    q = np.where(eff[..., None] != 0, q, 32)
    q = np.clip(q, 0, 63).astype(np.uint8).reshape(rows, nsb, 2, 4, 32)   # [h, r, l]
    ql = np.zeros((rows, nsb, 2, 2, 32), np.uint8)                       # [h, r % 2, l]
    ql |= q[:, :, :, 0:2, :] & 15
    ql |= (q[:, :, :, 2:4, :] & 15) << 4
    qh = np.zeros((rows, nsb, 2, 32), np.uint8)
    for r in range(4):
        qh |= (q[:, :, :, r, :] >> 4) << (2 * r)
    return np.concatenate([ql.reshape(rows, nsb, 128), qh.reshape(rows, nsb, 64),
                           sc.view(np.uint8).reshape(rows, nsb, 16), _f16_bytes(d32)],
                          axis=2).reshape(rows, -1)


def quantize(w: np.ndarray, qtype: str) -> np.ndarray:
    if qtype == Q8_0:
        return quantize_q8_0(w)
    if qtype == Q4_0:
        return quantize_q4_0(w)
    if qtype == Q4_1:
        return quantize_min_scale(w, 4)
    if qtype == Q5_0:
        return quantize_q5_0(w)
    if qtype == Q5_1:
        return quantize_min_scale(w, 5)
    if qtype == Q4_K:
        return quantize_q4_k(w)
    if qtype == Q6_K:
        return quantize_q6_k(w)
    raise ValueError(f"unknown qtype {qtype}")


# --------------------------------------------------------------------------
# layer inputs
# --------------------------------------------------------------------------
def gen_expert_pool(seed: int, n_experts: int, D: int, F: int, qtype: str,
                    std: float, threads: int | None = None):
    """Draw n_experts SwiGLU experts ~N(0, std) and encode them.

    Expert e draws from its own stream ``default_rng([seed, e])`` (gate, up,
    down in that order), so the bytes do not depend on the thread count.
    Returns (gate, up, down) uint8 arrays of shapes
    [n, F, D/32*bs], [n, F, D/32*bs], [n, D, F/32*bs] (the pool layout).
    """
    gate = np.empty((n_experts, F, row_bytes(D, qtype)), np.uint8)
    up = np.empty_like(gate)
    down = np.empty((n_experts, D, row_bytes(F, qtype)), np.uint8)
    s32 = np.float32(std)

    def one(e):
        r = np.random.default_rng([seed, e])
        gate[e] = quantize(r.standard_normal((F, D), np.float32) * s32, qtype)
        up[e] = quantize(r.standard_normal((F, D), np.float32) * s32, qtype)
        down[e] = quantize(r.standard_normal((D, F), np.float32) * s32, qtype)

    if threads is None:
        threads = min(32, os.cpu_count() or 1)
    if threads <= 1 or n_experts == 1:
        for e in range(n_experts):
            one(e)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(one, range(n_experts)))
    return gate, up, down


def zipf_bias(rng: np.random.Generator, E: int, s: float) -> np.ndarray:
    """Per-expert router bias b_e = ln p_e with p_e proportional to rank_e^-s
    over a random ranking of the experts (skews expert loads)."""
    rank = rng.permutation(E) + 1
    p = rank.astype(np.float64) ** (-s)
    p /= p.sum()
    return np.log(p).astype(np.float32)


def locality_trace(rng: np.random.Generator, T: int, E: int, k: int,
                   repeat: float = 0.8):
    """Routing logits [T, E] whose top-k follows a temporal-locality trace.

    Token 0 takes a uniform k-subset.  Token t keeps
    n_rep = floor(repeat*k) + Bernoulli(frac(repeat*k)) experts drawn uniformly
    from token t-1's set and draws the rest uniformly from the other experts.
    The logits of each token are E draws of N(0,1), sorted, the k largest
    given to the chosen set in random order and the rest to the others in
    random order, so the top-k of the row is exactly the chosen set.
    Returns (logits float32 [T, E], sets int32 [T, k]).
    """
    base = repeat * k
    n_lo = int(math.floor(base))
    frac = base - n_lo
    logits = np.empty((T, E), np.float32)
    sets = np.empty((T, k), np.int32)
    prev = None
    for t in range(T):
        if prev is None:
            cur = rng.choice(E, size=k, replace=False)
        else:
            n_rep = n_lo + int(rng.random() < frac)
            n_rep = min(n_rep, k)
            keep = rng.choice(prev, size=n_rep, replace=False)
            others = np.setdiff1d(np.arange(E), prev, assume_unique=False)
            new = rng.choice(others, size=k - n_rep, replace=False)
            cur = np.concatenate([keep, new])
        vals = np.sort(rng.standard_normal(E).astype(np.float32))[::-1]
        row = np.empty(E, np.float32)
        rest = np.setdiff1d(np.arange(E), cur)
        row[rng.permutation(cur)] = vals[:k]
        row[rng.permutation(rest)] = vals[k:]
        logits[t] = row
        sets[t] = cur
        prev = cur
    return logits, sets


@dataclass
class LayerInputs:
    cfg: LayerConfig
    x: np.ndarray                 # [T, D] float32 values (exact for bf16)
    x_raw: np.ndarray             # bytes the GPU reads: float32 or uint16 bf16 bits
    w_router: np.ndarray | None   # [D, E] float32
    bias: np.ndarray | None       # [E] float32
    logits: np.ndarray | None     # [T, E] float32 when routing comes from a trace
    gate: np.ndarray              # pool bytes (see gen_expert_pool)
    up: np.ndarray
    down: np.ndarray
    shared: tuple | None          # (gate, up, down) with one expert, cfg.shared_qtype


def gen_activations(rng: np.random.Generator, T: int, D: int, dtype: str):
    x = rng.standard_normal((T, D), np.float32)
    if dtype == "bf16":
        raw = f32_to_bf16_bits(x)
        return bf16_bits_to_f32(raw), raw
    return x, x.copy()


def make_layer(cfg: LayerConfig, T: int | None = None, seed: int | None = None,
               experts: bool = True) -> LayerInputs:
    """All inputs of one layer call, deterministic in (cfg, T, seed)."""
    T = cfg.T if T is None else T
    seed = cfg.seed if seed is None else seed
    rng = np.random.default_rng([seed, 0x5EED, T])
    if experts:
        gate, up, down = gen_expert_pool(seed, cfg.E, cfg.D, cfg.F, cfg.qtype, cfg.expert_std)
    else:
        gate = up = down = None
    shared = None
    if cfg.shared_F:
        shared = gen_expert_pool(seed + 7777, 1, cfg.D, cfg.shared_F, cfg.shared_qtype,
                                 cfg.expert_std)
    w_router = bias = logits = None
    if cfg.logits_from_trace:
        logits, _ = locality_trace(rng, T, cfg.E, cfg.k)
    else:
        w_router = (rng.standard_normal((cfg.D, cfg.E), np.float32)
                    * np.float32(cfg.router_std))
        if cfg.zipf_s is not None:
            bias = zipf_bias(rng, cfg.E, cfg.zipf_s)
    x, x_raw = gen_activations(rng, T, cfg.D, cfg.x_dtype)
    return LayerInputs(cfg, x, x_raw, w_router, bias, logits, gate, up, down, shared)
