"""Pins of the CPU oracle against facts fixed outside it.

Each test checks the oracle against something other than itself: the IEEE
binary16 definition, hand-packed blocks with closed-form values, numpy's own
routines on special cases, brute force on tiny inputs, invariants, or a
hand-worked LRU trace.  A plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, a swapped nibble) fails one of them.
"""
import itertools
import os

import numpy as np
import pytest

import synthetic as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- fp16 scale
@pytest.mark.parametrize("bits,val", [
    (0x3C00, 1.0), (0xC000, -2.0), (0x3555, 0.333251953125), (0x7BFF, 65504.0),
    (0x0001, 2.0 ** -24), (0x03FF, 1023 * 2.0 ** -24), (0x0400, 2.0 ** -14),
    (0x8000, -0.0), (0x5A00, 192.0), (0xB400, -0.25),
])
def test_half_to_double_known_patterns(orc, bits, val):
    assert orc.half_to_double(bits) == val


def test_half_to_double_matches_numpy_all_finite(orc):
    # every finite binary16 pattern against numpy's own float16 conversion
    for bits in range(0, 0x10000, 7):
        ref = float(np.array([bits], np.uint16).view(np.float16)[0])
        got = orc.half_to_double(bits)
        if np.isnan(ref):
            assert np.isnan(got)
        else:
            assert got == ref, hex(bits)


# ---------------------------------------------------------- hand-packed blocks
def _golden_blocks():
    out = []
    with open(os.path.join(GOLDEN, "blocks.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            parts = line.split()
            out.append((parts[0], parts[1], bytes.fromhex(parts[2]),
                        np.array([float(v) for v in parts[3:]])))
    return out


@pytest.mark.parametrize("name,qtype,raw,vals", _golden_blocks(),
                         ids=[b[0] for b in _golden_blocks()])
def test_dequant_hand_packed_blocks(orc, name, qtype, raw, vals):
    assert len(raw) == S.BLOCK_BYTES[qtype] == orc.block_bytes(qtype)
    n = S.BLOCK_WEIGHTS[qtype]
    assert len(vals) == n == orc.block_weights(qtype)
    got = orc.dequant_row(np.frombuffer(raw, np.uint8), qtype, n)
    np.testing.assert_array_equal(got, vals)


@pytest.mark.parametrize("qtype", ["q8_0", "q4_0", "q4_1", "q5_0", "q5_1", "q4_k", "q6_k"])
def test_dequant_row_of_several_blocks_keeps_block_order(orc, qtype):
    blocks = [b for b in _golden_blocks() if b[1] == qtype]
    assert len(blocks) >= 2
    raw = b"".join(b[2] for b in blocks)
    got = orc.dequant_row(np.frombuffer(raw, np.uint8), qtype,
                          S.BLOCK_WEIGHTS[qtype] * len(blocks))
    np.testing.assert_array_equal(got, np.concatenate([b[3] for b in blocks]))


@pytest.mark.parametrize("qtype,slack,top", [("q8_0", 127, 127), ("q4_0", 8, 7),
                                             ("q5_0", 16, 15)])
def test_quantizer_roundtrip_error_bound(orc, qtype, slack, top):
    # encoder (input generator) + decoder (oracle): |w - dequant(w)| <= |d|/2
    # up to the fp16 rounding of d (relative 2^-11, times the largest code),
    # except where the code clips at the top of the range: Q4_0 codes span
    # [-8, 7] * d, so a weight of the opposite sign to the block's largest
    # one can exceed 7.5|d| and lands on 7d (error |w| - 7|d| <= |d|).
    rng = np.random.default_rng(5)
    w = (rng.standard_normal((16, 256)) * 0.02).astype(np.float32)
    w[3, 32:64] = 0.0                      # an all-zero block
    packed = S.quantize(w, qtype)
    deq = orc.dequant_matrix(packed, qtype, 256)
    bs = S.BLOCK_BYTES[qtype]
    d16 = np.abs(packed.reshape(16, 8, bs)[:, :, :2].copy().view(np.float16)[..., 0]
                 .astype(np.float64))
    dd = np.repeat(d16, 32, axis=1)
    bound = np.maximum(0.5 * dd, np.abs(w) - top * dd) + slack * 2.0 ** -11 * dd + 1e-12
    assert np.all(np.abs(deq - w) <= bound)
    assert np.all(np.abs(deq - w) <= dd * (1 + slack * 2.0 ** -11) + 1e-12)
    assert np.all(deq[3, 32:64] == 0.0)


@pytest.mark.parametrize("qtype,top", [("q4_1", 15), ("q5_1", 31)])
def test_min_scale_quantizer_roundtrip_error_bound(orc, qtype, top):
    # value = q * d + m with m = the block minimum and d = range / top: the
    # error is at most d/2, plus the fp16 rounding of d (relative 2^-11,
    # times the code) and of m (relative 2^-11); the block minimum itself
    # lands on code 0 and decodes to fp16(m).
    rng = np.random.default_rng(15)
    w = (rng.standard_normal((16, 256)) * 0.02 + 0.003).astype(np.float32)
    w[5, 64:96] = 0.0125                    # a constant block: d = 0, q = 0
    packed = S.quantize(w, qtype)
    deq = orc.dequant_matrix(packed, qtype, 256)
    blk = packed.reshape(16, 8, S.BLOCK_BYTES[qtype])
    d16 = blk[:, :, 0:2].copy().view(np.float16)[..., 0].astype(np.float64)
    m16 = blk[:, :, 2:4].copy().view(np.float16)[..., 0].astype(np.float64)
    assert np.all(d16 >= 0)
    dd = np.repeat(d16, 32, axis=1)
    mm = np.repeat(np.abs(m16), 32, axis=1)
    bound = 0.5 * dd * (1 + 2.0 ** -10) + top * 2.0 ** -11 * dd + 2.0 ** -11 * mm + 1e-12
    assert np.all(np.abs(deq - w) <= bound)
    wb = w.reshape(16, 8, 32)
    imin = np.argmin(wb, axis=2)
    got = deq.reshape(16, 8, 32)[np.arange(16)[:, None], np.arange(8)[None], imin]
    np.testing.assert_array_equal(got, m16)
    np.testing.assert_array_equal(deq[5, 64:96], np.float64(np.float16(0.0125)))


def test_q5_0_largest_weight_lands_on_code_zero(orc):
    rng = np.random.default_rng(16)
    w = (rng.standard_normal((4, 64)) * 0.02).astype(np.float32)
    packed = S.quantize(w, "q5_0").reshape(4, 2, 22)
    wb = w.reshape(4, 2, 32)
    deq = orc.dequant_matrix(packed.reshape(4, -1), "q5_0", 64).reshape(4, 2, 32)
    for r in range(4):
        for b in range(2):
            i = int(np.argmax(np.abs(wb[r, b])))
            word = int.from_bytes(bytes(packed[r, b, 2:6]), "little")
            code = ((packed[r, b, 6 + i % 16] >> (0 if i < 16 else 4)) & 0xF) | \
                (((word >> i) & 1) << 4)
            assert code == 0
            d16 = float(packed[r, b, :2].copy().view(np.float16)[0])
            assert deq[r, b, i] == -16 * d16


@pytest.mark.parametrize("qtype", ["q4_k", "q6_k"])
def test_k_quant_encoder_roundtrip_bound(orc, qtype):
    # encoder (input generator) + decoder (oracle).  Q6_K: |w - v| <= |d sc|/2
    # where the code does not clip; Q4_K: <= d sc/2 inside the sub-block's
    # range, and in any case <= d sc/2 + 7.5 d + dmin/2 (rounding the scale
    # and the min to integers moves the range's ends by at most that); fp16
    # slack on top
    rng = np.random.default_rng(17)
    w = (rng.standard_normal((8, 512)) * 0.02).astype(np.float32)
    w[2, 256:512] = 0.0                                     # an all-zero super-block
    packed = S.quantize(w, qtype)
    deq = orc.dequant_matrix(packed, qtype, 512)
    blk = packed.reshape(8, 2, S.BLOCK_BYTES[qtype])
    if qtype == "q4_k":
        d = blk[..., 0:2].copy().view(np.float16)[..., 0].astype(np.float64)
        dmin = blk[..., 2:4].copy().view(np.float16)[..., 0].astype(np.float64)
        # d sc/2 <= 31.5 d for sc <= 63
        bound = np.repeat(39.5 * d + 0.5 * dmin, 256, axis=1) + 2.0 ** -9 * np.abs(w) + 1e-9
        assert np.all(np.abs(deq - w) <= bound)
    else:
        d = blk[..., 208:210].copy().view(np.float16)[..., 0].astype(np.float64)
        sc = blk[..., 192:208].copy().view(np.int8).astype(np.float64)     # [8, 2, 16]
        eff = np.abs(d[..., None] * sc).reshape(8, 32)
        step = np.repeat(eff, 16, axis=1)
        assert np.all(np.abs(deq - w) <= np.maximum(0.5 * step, np.abs(w) - 31 * step)
                      + 2.0 ** -9 * np.abs(w) + 1e-9)
    assert np.all(deq[2, 256:512] == 0.0)
    assert np.abs(deq - w).max() < 0.25 * np.abs(w).max()


def test_q4_0_largest_weight_lands_on_code_zero(orc):
    rng = np.random.default_rng(6)
    w = (rng.standard_normal((4, 64)) * 0.02).astype(np.float32)
    packed = S.quantize_q4_0(w).reshape(4, 2, 18)
    deq = orc.dequant_matrix(packed.reshape(4, -1), "q4_0", 64).reshape(4, 2, 32)
    wb = w.reshape(4, 2, 32)
    for r in range(4):
        for b in range(2):
            i = np.argmax(np.abs(wb[r, b]))
            code = (packed[r, b, 2 + i % 16] >> (0 if i < 16 else 4)) & 0xF
            assert code == 0
            d16 = float(packed[r, b, :2].copy().view(np.float16)[0])
            assert abs(deq[r, b, i] - wb[r, b, i]) <= 8 * abs(d16) * 2.0 ** -10


# --------------------------------------------------------------- router logits
def test_router_logits_against_numpy_matmul(orc):
    rng = np.random.default_rng(7)
    x = rng.standard_normal((5, 64)).astype(np.float32)
    w = (rng.standard_normal((64, 12)) * 0.05).astype(np.float32)
    b = rng.standard_normal(12).astype(np.float32)
    ref = (x.astype(np.float64) @ w.astype(np.float64) + b).astype(np.float32)
    np.testing.assert_array_equal(orc.router_logits(x, w, b), ref)


def test_router_logits_identity_router_returns_x(orc):
    x = np.arange(24, dtype=np.float32).reshape(3, 8) / 7
    np.testing.assert_array_equal(orc.router_logits(x, np.eye(8, dtype=np.float32)), x)


# ---------------------------------------------------------- top-k and gates
def test_topk_brute_force_all_subsets(orc):
    rng = np.random.default_rng(8)
    for E, k in [(5, 2), (6, 3), (7, 1), (8, 4), (6, 6)]:
        L = rng.standard_normal((20, E)).astype(np.float32)
        ids, g = orc.select(L, k)
        for t in range(20):
            best = max(itertools.combinations(range(E), k),
                       key=lambda s: sum(float(L[t, i]) for i in s))
            assert set(ids[t]) == set(best)
            assert list(L[t, ids[t]]) == sorted(L[t, ids[t]], reverse=True)


def test_topk_ties_go_to_lower_index(orc):
    L = np.array([[1, 3, 3, 2, 3], [0, 0, 0, 0, 0], [5, 4, 5, 4, 5]], np.float32)
    ids, _ = orc.select(L, 3)
    np.testing.assert_array_equal(ids, [[1, 2, 4], [0, 1, 2], [0, 2, 4]])


def test_gates_are_softmax_of_selected_logits(orc):
    rng = np.random.default_rng(9)
    L = (rng.standard_normal((50, 32)) * 3).astype(np.float32)
    ids, g = orc.select(L, 6)
    sel = np.take_along_axis(L.astype(np.float64), ids, axis=1)
    ref = np.exp(sel - sel.max(axis=1, keepdims=True))
    ref /= ref.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(g, ref, rtol=1e-12, atol=0)
    assert np.all(np.abs(g.sum(axis=1) - 1) <= 1e-12)
    assert np.all(np.diff(g, axis=1) <= 0)    # descending logits -> descending gates


def test_gates_without_renorm_are_full_softmax(orc):
    rng = np.random.default_rng(10)
    L = rng.standard_normal((10, 16)).astype(np.float32)
    ids, g = orc.select(L, 4, renorm=False)
    p = np.exp(L.astype(np.float64) - L.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(g, np.take_along_axis(p, ids, axis=1), rtol=1e-12)
    ids_all, g_all = orc.select(L, 16)
    np.testing.assert_allclose(g_all.sum(axis=1), 1.0, rtol=0, atol=1e-12)


def test_near_tie_detector(orc):
    L = np.array([[3.0, 2.0, 1.0, 0.0],
                  [3.0, 2.0, 2.0 - 5e-6, 0.0],     # k-th vs (k+1)-th gap
                  [3.0, 3.0 - 2e-6, 1.0, 0.0]],    # gap inside the top-k
                 np.float32)
    np.testing.assert_array_equal(orc.near_tie_tokens(L, 2), [1, 2])


# ---------------------------------------------------------------- permutation
@pytest.mark.parametrize("T,k,E", [(1, 1, 1), (4, 2, 8), (37, 8, 128), (300, 10, 512)])
def test_permutation_invariants(orc, T, k, E):
    rng = np.random.default_rng(T)
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, perm, inv = orc.permute(ids, E)
    flat = ids.ravel()
    np.testing.assert_array_equal(counts, np.bincount(flat, minlength=E))
    assert offsets[0] == 0 and offsets[-1] == T * k
    assert np.all(np.diff(offsets) == counts)
    np.testing.assert_array_equal(perm[inv], np.arange(T * k))
    np.testing.assert_array_equal(inv[perm], np.arange(T * k))
    # library stable sort gives the same order (expert, then t, then j)
    np.testing.assert_array_equal(perm, np.argsort(flat, kind="stable"))
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.all(flat[seg] == e) and np.all(np.diff(seg) > 0)


# ------------------------------------------------------------------ the layer
def _textbook_swiglu(x, Wg, Wu, Wd):
    a = x @ Wg.T
    u = x @ Wu.T
    h = a / (1.0 + np.exp(-a)) * u
    return h @ Wd.T


# integer value range of each type at scale 1 (and, for the _1 types, the
# fp16 minimum m = -8 / -16 that centres it), and the code offset
_INT_RANGE = {"q8_0": (-20, 21), "q4_0": (-8, 8), "q4_1": (-8, 8),
              "q5_0": (-16, 16), "q5_1": (-16, 16), "q4_k": (-8, 8), "q6_k": (-32, 32)}
_CODE_OFF = {"q4_0": 8, "q4_1": 8, "q5_0": 16, "q5_1": 16}
_MIN_BITS = {"q4_1": 0xC800, "q5_1": 0xCC00}      # fp16 -8.0, -16.0


def _pack_int_matrix_k(codes, qtype):
    """K-quant packing of an integer matrix, by the format definition: Q4_K
    with d = dmin = 1, every sub-block scale 1 and min 8 (value = code - 8);
    Q6_K with d = 1 and every scale 1 (value = code - 32)."""
    rows, cols = codes.shape
    nsb = cols // 256
    c = codes.reshape(rows, nsb, 256).astype(np.int64)
    out = np.zeros((rows, nsb, S.BLOCK_BYTES[qtype]), np.uint8)
    if qtype == "q4_k":
        q = c + 8
        assert q.min() >= 0 and q.max() < 16
        out[..., 0:4] = [0x00, 0x3C, 0x00, 0x3C]              # d = dmin = 1.0
        out[..., 4:8] = 1                                      # sc_0..3 = 1
        out[..., 8:12] = 8                                     # m_0..3 = 8
        out[..., 12:16] = 1 | (8 << 4)                         # sc_4..7 = 1, m_4..7 = 8
        for ch in range(4):
            out[..., 16 + 32 * ch:16 + 32 * ch + 32] = (
                q[..., 64 * ch:64 * ch + 32] | (q[..., 64 * ch + 32:64 * ch + 64] << 4))
    else:
        q = c + 32
        assert q.min() >= 0 and q.max() < 64
        for i in range(256):
            h, r, l = i // 128, (i % 128) // 32, i % 32
            out[..., 64 * h + 32 * (r % 2) + l] |= ((q[..., i] & 15) << (4 * (r // 2))).astype(np.uint8)
            out[..., 128 + 32 * h + l] |= ((q[..., i] >> 4) << (2 * r)).astype(np.uint8)
        out[..., 192:208] = 1                                  # scales = 1
        out[..., 208:210] = [0x00, 0x3C]                       # d = 1.0
    return out.reshape(rows, -1)


def _pack_int_matrix(codes, qtype, dbits=0x3C00):
    """Pack an integer matrix with scale 1.0 in every block (test-side
    packing by the format definition; values = codes).  The _1 types get
    m = -offset so that code = value + offset as in their _0 twins."""
    if qtype in ("q4_k", "q6_k"):
        return _pack_int_matrix_k(codes, qtype)
    rows, cols = codes.shape
    nb = cols // 32
    lo = codes.reshape(rows, nb, 32).astype(np.int64)
    fields = [np.full((rows, nb, 2), [dbits & 0xFF, dbits >> 8], np.uint8)]
    if qtype == "q8_0":
        fields.append((lo & 0xFF).astype(np.uint8))
    else:
        c = (lo + _CODE_OFF[qtype]).astype(np.uint32)
        assert c.min() >= 0 and c.max() < 2 * _CODE_OFF[qtype]
        if qtype in _MIN_BITS:
            mb = _MIN_BITS[qtype]
            fields.append(np.full((rows, nb, 2), [mb & 0xFF, mb >> 8], np.uint8))
        if qtype in ("q5_0", "q5_1"):
            word = np.zeros((rows, nb), np.uint64)
            for i in range(32):
                word |= ((c[..., i] >> 4) & 1).astype(np.uint64) << np.uint64(i)
            fields.append(np.stack([(word >> np.uint64(8 * j)) & np.uint64(0xFF)
                                    for j in range(4)], axis=-1).astype(np.uint8))
        n = c & 0xF
        fields.append((n[..., :16] | (n[..., 16:] << 4)).astype(np.uint8))
    return np.concatenate(fields, axis=2).reshape(rows, -1)


def test_int_matrix_packer_agrees_with_the_golden_layouts(orc):
    # the packer above against the hand-packed golden blocks' layouts: a
    # unit-scale block of codes 0..31 (values code - offset) decodes to them
    for qt in ("q4_0", "q4_1", "q5_0", "q5_1", "q8_0", "q4_k", "q6_k"):
        lo, hi = _INT_RANGE[qt]
        n = S.BLOCK_WEIGHTS[qt]
        vals = (np.arange(n) * 7) % (hi - lo) + lo
        raw = _pack_int_matrix(vals[None], qt)
        assert raw.shape[1] == S.BLOCK_BYTES[qt]
        np.testing.assert_array_equal(orc.dequant_row(raw[0], qt, n), vals)


@pytest.mark.parametrize("qtype", ["q8_0", "q4_0", "q4_1", "q5_0", "q5_1", "q4_k", "q6_k"])
def test_single_expert_is_textbook_swiglu(orc, qtype):
    # integer-valued weights (scale 1) so the dequantized matrices are known
    # exactly; E=1, k=1 reduces the layer to a plain SwiGLU FFN.
    rng = np.random.default_rng(11)
    D, F = (256, 512) if qtype in ("q4_k", "q6_k") else (64, 96)
    lo, hi = _INT_RANGE[qtype]
    Wg = rng.integers(lo, hi, (F, D))
    Wu = rng.integers(lo, hi, (F, D))
    Wd = rng.integers(lo, hi, (D, F))
    x = (rng.integers(-3, 4, (3, D)) / 16).astype(np.float32)
    gate = _pack_int_matrix(Wg, qtype)[None]
    up = _pack_int_matrix(Wu, qtype)[None]
    down = _pack_int_matrix(Wd, qtype)[None]
    ids = np.zeros((3, 1), np.int32)
    g = np.ones((3, 1))
    y = orc.layer(x, ids, g, gate, up, down, qtype, F)
    ref = _textbook_swiglu(x.astype(np.float64), Wg.astype(float), Wu.astype(float), Wd.astype(float))
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-9 * np.abs(ref).max())


def test_routed_layer_is_gate_weighted_sum_of_single_experts(orc):
    cfg = S.CONFIGS["tiny"]
    L = S.make_layer(cfg)
    _, ids, g = orc.route(L.x, L.w_router, None, cfg.k)
    y = orc.layer(L.x, ids, g, L.gate, L.up, L.down, cfg.qtype, cfg.F)
    for t in range(cfg.T):
        acc = np.zeros(cfg.D)
        for j in range(cfg.k):
            e = ids[t, j]
            ye = orc.layer(L.x[t:t + 1], np.zeros((1, 1), np.int32), np.ones((1, 1)),
                           L.gate[e:e + 1], L.up[e:e + 1], L.down[e:e + 1], cfg.qtype, cfg.F)
            acc += g[t, j] * ye[0]
        np.testing.assert_allclose(y[t], acc, rtol=1e-12, atol=1e-15)


def test_dense_masked_equals_routed(orc):
    cfg = S.CONFIGS["tiny"]
    L = S.make_layer(cfg)
    _, ids, g = orc.route(L.x, L.w_router, None, cfg.k)
    y = orc.layer(L.x, ids, g, L.gate, L.up, L.down, cfg.qtype, cfg.F)
    yd = orc.layer(L.x, ids, g, L.gate, L.up, L.down, cfg.qtype, cfg.F, dense=True)
    assert np.abs(y - yd).max() <= 1e-12 * np.abs(y).max()


def test_dequantized_dense_evaluation_matches_layer(orc):
    # dequantize each expert with the pinned block decoder and evaluate the
    # textbook FFN with numpy; must equal the oracle's routed layer
    cfg = S.CONFIGS["tiny"]
    L = S.make_layer(cfg)
    _, ids, g = orc.route(L.x, L.w_router, None, cfg.k)
    y = orc.layer(L.x, ids, g, L.gate, L.up, L.down, cfg.qtype, cfg.F)
    x64 = L.x.astype(np.float64)
    ref = np.zeros_like(y)
    for t in range(cfg.T):
        for j in range(cfg.k):
            e = ids[t, j]
            Wg = orc.dequant_matrix(L.gate[e], cfg.qtype, cfg.D)
            Wu = orc.dequant_matrix(L.up[e], cfg.qtype, cfg.D)
            Wd = orc.dequant_matrix(L.down[e], cfg.qtype, cfg.F)
            ref[t] += g[t, j] * _textbook_swiglu(x64[t:t + 1], Wg, Wu, Wd)[0]
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-12 * np.abs(ref).max())


def test_shared_expert_adds_with_weight_one(orc):
    rng = np.random.default_rng(12)
    D, F, E, k, sF = 64, 64, 4, 2, 32
    gate, up, down = S.gen_expert_pool(3, E, D, F, "q4_0", 0.05, threads=1)
    shared = S.gen_expert_pool(4, 1, D, sF, "q8_0", 0.05, threads=1)
    x = rng.standard_normal((3, D)).astype(np.float32)
    ids = np.array([[0, 1], [2, 3], [1, 2]], np.int32)
    g = np.array([[0.7, 0.3], [0.5, 0.5], [0.9, 0.1]])
    y0 = orc.layer(x, ids, g, gate, up, down, "q4_0", F)
    y1 = orc.layer(x, ids, g, gate, up, down, "q4_0", F, shared=shared)
    ys = orc.layer(x, np.zeros((3, 1), np.int32), np.ones((3, 1)), *shared, "q8_0", sF)
    np.testing.assert_allclose(y1, y0 + ys, rtol=1e-12, atol=1e-15)


def test_token_subset_and_expert_rows(orc):
    cfg = S.CONFIGS["tiny"]
    L = S.make_layer(cfg)
    _, ids, g = orc.route(L.x, L.w_router, None, cfg.k)
    y = orc.layer(L.x, ids, g, L.gate, L.up, L.down, cfg.qtype, cfg.F)
    ys = orc.layer(L.x, ids, g, L.gate, L.up, L.down, cfg.qtype, cfg.F, tokens=[3, 1])
    np.testing.assert_array_equal(ys, y[[3, 1]])
    counts, offsets, perm, inv = orc.permute(ids, cfg.E)
    Y = orc.expert_rows(L.x, perm, offsets, cfg.k, L.gate, L.up, L.down, cfg.qtype, cfg.F)
    comb = np.zeros_like(y)
    for t in range(cfg.T):
        for j in range(cfg.k):
            comb[t] += g[t, j] * Y[inv[t * cfg.k + j]]
    np.testing.assert_allclose(comb, y, rtol=1e-12, atol=1e-15)


# ------------------------------------------------------------------ LRU cache
def test_lru_hand_worked_trace(orc):
    # E=6 experts, 3 slots; every requested expert is stamped with the step
    # number (1, 2, ...).  Worked by hand from the replacement rules:
    #  1: [0,1] both miss, empty slots 0,1             stamps 0@1 1@1
    #  2: [1,2] 1 hits; 2 takes empty slot 2            1@2 2@2
    #  3: [3]   no empty slot; oldest unrequested is 0  -> slot 0, evicts 0
    #  4: [1,4] 1 hits; 4: oldest unrequested is 2@2 (3@3 is newer) -> slot 2
    #  5: [5,0] 5: oldest of {3@3, 1@4, 4@4} is 3 -> slot 0;
    #           0: 1@4 and 4@4 tie -> lower expert id 1 -> slot 1
    c = orc.LRU(6, 3)
    steps = [
        ([0, 1], [0, 1], [True, True], [-1, -1]),
        ([1, 2], [1, 2], [False, True], [-1, -1]),
        ([3], [0], [True], [0]),
        ([1, 4], [1, 2], [False, True], [-1, 2]),
        ([5, 0], [0, 1], [True, True], [3, 1]),
    ]
    for req, slots, misses, ev in steps:
        s, m, e = c.request(np.array(req, np.int32))
        assert list(s) == slots and list(m) == misses and list(e) == ev, req


def test_lru_wanted_expert_is_never_evicted(orc):
    c = orc.LRU(5, 2)
    c.request([1])          # 1@1 -> slot 0
    c.request([0])          # 0@2 -> slot 1
    # 1 is the least recently used but is requested again in this step, so
    # the miss on 4 must evict 0 instead
    s, m, e = c.request([4, 1])
    assert list(m) == [True, False] and list(e) == [0, -1] and list(s) == [1, 0]


def test_lru_capacity_and_bad_ids(orc):
    c = orc.LRU(8, 3)
    with pytest.raises(OverflowError):
        c.request([0, 1, 2, 3])
    with pytest.raises(ValueError):
        c.request([0, 0])
    with pytest.raises(ValueError):
        c.request([9])


def test_lru_invariants_random_trace(orc):
    rng = np.random.default_rng(13)
    E, n_slots, k = 32, 12, 8
    c = orc.LRU(E, n_slots)
    resident = {}
    total_miss = 0
    for step in range(200):
        req = rng.choice(E, k, replace=False).astype(np.int32)
        s, m, ev = c.request(req)
        for e, slot, miss, vic in zip(req, s, m, ev):
            assert miss == (e not in resident)
            if vic >= 0:
                assert vic not in req and resident.pop(vic) == slot
            resident[e] = slot
        assert len(resident) <= n_slots
        assert len(set(resident.values())) == len(resident)
        total_miss += int(m.sum())
    assert 0 < total_miss < 200 * k


# ----------------------------------------------------- global LRU + resize
def test_global_lru_hand_worked_trace(orc):
    # 2 layers x 4 experts, keys layer*4 + e; 4 slots, capacity 3 at start.
    # One step counter for every layer.  Worked by hand from the rules:
    #  1: L0 [0,1]   keys 0,1 -> empty slots 0,1                 0@1 1@1
    #  2: L1 [0]     key 4 -> empty slot 2                       4@2
    #  3: L0 [1,2]   1 hits (slot 1); key 2: full, oldest not requested
    #                is 0@1 (4@2 newer, 1 requested) -> slot 0, evicts 0
    #  4: L1 [1,0]   key 5: full; keys 4, 5 of layer 1 are protected;
    #                1@3 and 2@3 tie -> lower key 1 -> slot 1; key 4 hits
    #  resize(4):    one more empty slot (3)
    #  6: L0 [3]     key 3 -> empty slot 3                       3@5
    #  resize(2):    4 resident > 2: evict 2@3, then 4@4 and 5@4 tie -> 4;
    #                slot 3 (key 3) is >= 2 -> moves to empty slot 0
    #  8: L1 [1]     key 5 hits in slot 1
    #  9: L0 [0,1,2] more ids than the capacity
    # 10: L1 [2]     key 6: full; oldest not requested of 3@5, 5@6 -> 3
    g = orc.GlobalLRU(2, 4, 4, 3)
    chk = lambda r, s, m, e: (list(r[0]) == s and list(r[1]) == m and list(r[2]) == e) or r
    assert chk(g.request(0, [0, 1]), [0, 1], [True, True], [-1, -1]) is True
    assert chk(g.request(1, [0]), [2], [True], [-1]) is True
    assert chk(g.request(0, [1, 2]), [1, 0], [False, True], [-1, 0]) is True
    assert chk(g.request(1, [1, 0]), [1, 2], [True, False], [1, -1]) is True
    ev, mv = g.resize(4)
    assert len(ev) == 0 and len(mv) == 0
    assert chk(g.request(0, [3]), [3], [True], [-1]) is True
    ev, mv = g.resize(2)
    assert list(ev) == [2, 4] and mv.tolist() == [[3, 0]]
    assert chk(g.request(1, [1]), [1], [False], [-1]) is True
    with pytest.raises(OverflowError):
        g.request(0, [0, 1, 2])
    assert chk(g.request(1, [2]), [0], [True], [3]) is True
    with pytest.raises(ValueError):
        g.resize(5)
    with pytest.raises(ValueError):
        g.request(2, [0])


def test_global_lru_one_layer_is_the_per_layer_lru(orc):
    # with one layer and a fixed capacity the global rules are the per-layer
    # ones (pinned by its own hand-worked trace above)
    rng = np.random.default_rng(17)
    E, n_slots, k = 24, 9, 6
    a, b = orc.LRU(E, n_slots), orc.GlobalLRU(1, E, n_slots, n_slots)
    for step in range(300):
        req = rng.choice(E, k, replace=False).astype(np.int32)
        ra, rb = a.request(req), b.request(0, req)
        for x, y in zip(ra, rb):
            assert np.array_equal(x, y), step


def test_global_lru_invariants_random_trace_with_resizes(orc):
    rng = np.random.default_rng(19)
    L, E, max_slots, k = 4, 16, 40, 6
    g = orc.GlobalLRU(L, E, max_slots, 24)
    cap = 24
    where = {}                      # key -> slot
    for step in range(400):
        if step % 37 == 36:         # shrink or grow
            new = int(rng.integers(k, max_slots + 1))
            ev, mv = g.resize(new)
            if new >= cap:
                assert len(ev) == 0 and len(mv) == 0
            for key in ev:
                where.pop(int(key))
            old = dict(where)
            for src, dst in mv:
                key = [kk for kk, s in old.items() if s == src]
                assert len(key) == 1 and src >= new and dst < new
                where[key[0]] = int(dst)
            cap = new
            assert len(where) <= cap and all(s < cap for s in where.values())
            assert len(set(where.values())) == len(where)
        layer = int(rng.integers(L))
        req = rng.choice(E, k, replace=False).astype(np.int32)
        s, m, ev = g.request(layer, req)
        for e, slot, miss, vic in zip(req, s, m, ev):
            key = layer * E + int(e)
            assert miss == (key not in where)
            if vic >= 0:
                assert not (vic // E == layer and vic % E in req)
                assert where.pop(int(vic)) == slot
            where[key] = int(slot)
        assert len(where) <= cap and all(sl < cap for sl in where.values())
        assert len(set(where.values())) == len(where)


# ------------------------------------------------------- 8-bit activations
# Hand-worked blocks: with amax = 127 the scale is 1 and the codes are the
# values rounded half away from zero; with amax = 254 (scale 2, 1/scale = 0.5)
# and amax = 63.5 (scale 0.5, 1/scale = 2) every product is exact in fp32,
# so the codes below follow from the rounding rule alone.
ACT8_CASES = [
    # values (rest of the 32 zero), scale, codes
    ([63.5, -63.5, 0.5, -0.5, 1.49, -1.5, 2.5, 126.5, -127.0, 127.0], 1.0,
     [64, -64, 1, -1, 1, -2, 3, 127, -127, 127]),
    ([254.0, 3.0, -3.0, 5.0, 1.0, -1.0, 100.9, -0.9], 2.0,
     [127, 2, -2, 3, 1, -1, 50, 0]),
    ([63.5, 0.25, -0.25, 0.2, 31.75, -63.5], 0.5,
     [127, 1, -1, 0, 64, -127]),
    ([], 0.0, []),                                   # all zero: scale 0, codes 0
]


@pytest.mark.parametrize("vals,scale,codes", ACT8_CASES)
def test_act8_hand_worked_blocks(orc, vals, scale, codes):
    v = np.zeros(32, np.float32)
    v[:len(vals)] = vals
    q, d = orc.quantize_act8(v[None])
    assert d[0, 0] == np.float32(scale)
    want = np.zeros(32, np.int8)
    want[:len(codes)] = codes
    np.testing.assert_array_equal(q[0], want)


def test_act8_invariants(orc):
    rng = np.random.default_rng(23)
    v = (rng.standard_normal((64, 128)) * rng.uniform(0.01, 10, (64, 1))).astype(np.float32)
    q, d = orc.quantize_act8(v)
    vb, qb = v.reshape(64, 4, 32), q.reshape(64, 4, 32).astype(np.int64)
    assert np.abs(qb).max() <= 127
    # the largest magnitude of each block takes code +-127 with its sign
    i = np.abs(vb).argmax(axis=2)
    top = np.take_along_axis(qb, i[..., None], 2)[..., 0]
    np.testing.assert_array_equal(np.abs(top), 127)
    assert np.all(np.sign(top) == np.sign(np.take_along_axis(vb, i[..., None], 2)[..., 0]))
    # round trip within half a step (plus the fp32 rounding of 1/d and v/d)
    err = np.abs(qb * d[..., None].astype(np.float64) - vb)
    assert np.all(err <= 0.5 * d[..., None] * (1 + 2.0 ** -20) + 1e-30)
    # odd symmetry and power-of-two scale invariance
    qn, dn = orc.quantize_act8(-v)
    np.testing.assert_array_equal(qn, -q)
    np.testing.assert_array_equal(dn, d)
    q4, d4 = orc.quantize_act8(v * np.float32(4))
    np.testing.assert_array_equal(q4, q)
    np.testing.assert_array_equal(d4, d * np.float32(4))


def test_a8_layer_is_the_a16_layer_when_quantization_is_exact(orc):
    # x: block 0 holds 127 (scale 1), block 1 holds 254 and 2 (scale 2, codes
    # 127 and 1): both exact.  Gate rows read x_0 only (a = 127 * 127 =
    # 16129, where silu(a) = a in double), up rows read x_32 with weight c_r
    # in {-1, 0, 1} (u = 254 c_r), so h_r = 4096766 c_r = 127 * 32258 c_r:
    # every h block has scale 32258 (or 0) and codes 127 c_r exactly.  Then
    # the 8-bit-activation layer equals the 16-bit one in double.
    D, F = 64, 64
    x = np.zeros((1, D), np.float32)
    x[0, 0], x[0, 32], x[0, 33] = 127, 254, 2
    rng = np.random.default_rng(29)
    Wg = np.zeros((F, D), np.int64)
    Wg[:, 0] = 127
    Wu = np.zeros((F, D), np.int64)
    c = rng.integers(-1, 2, F)
    c[:32] = np.where(c[:32] == 0, 1, c[:32])       # block 0 of h is not all zero
    Wu[:, 32] = c
    Wd = rng.integers(-3, 4, (D, F))
    gate, up, down = (_pack_int_matrix(W, "q8_0")[None] for W in (Wg, Wu, Wd))
    ids, g = np.zeros((1, 1), np.int32), np.ones((1, 1))
    y16 = orc.layer(x, ids, g, gate, up, down, "q8_0", F)
    y8, b8 = orc.layer_a8(x, ids, g, gate, up, down, "q8_0", F, eps=1e-3, want_bound=True)
    np.testing.assert_array_equal(y8, y16)
    np.testing.assert_array_equal(b8, 0.0)
    assert np.abs(y16).max() > 1e8                   # not a trivial zero


def test_a8_layer_stays_within_the_quantization_error_of_the_a16_layer(orc):
    # With x on its own 8-bit grid the gate/up part is exact, and the down
    # projection is linear: y8 - y16 = sum_j g_j W_down (h^ - h) with
    # |h^_f - h_f| <= dh_b / 2 (+ the fp32 rounding of h), dh_b = max|h_b|/127
    # (h recomputed here with numpy from the dequantized weights).
    cfg = S.LayerConfig("a8", T=3, D=256, E=4, k=2, F=256, qtype="q8_0", x_dtype="f32",
                        y_dtype="f32", seed=31)
    L = S.make_layer(cfg)
    # put x on its own 8-bit grid: q * d is exactly representable
    q, d = orc.quantize_act8(L.x)
    xg = (q.reshape(3, 8, 32).astype(np.float32) * d[..., None]).reshape(3, 256)
    _, ids, g = orc.route(xg, L.w_router, None, cfg.k)
    y16 = orc.layer(xg, ids, g, L.gate, L.up, L.down, "q8_0", cfg.F)
    y8 = orc.layer_a8(xg, ids, g, L.gate, L.up, L.down, "q8_0", cfg.F)
    Wd = [orc.dequant_matrix(L.down[e], "q8_0", cfg.F) for e in range(cfg.E)]
    for t in range(3):
        bound = np.zeros(cfg.D)
        for j in range(cfg.k):
            e = ids[t, j]
            Wg = orc.dequant_matrix(L.gate[e], "q8_0", cfg.D)
            Wu = orc.dequant_matrix(L.up[e], "q8_0", cfg.D)
            a, u = Wg @ xg[t].astype(np.float64), Wu @ xg[t].astype(np.float64)
            h = a / (1 + np.exp(-a)) * u
            step = np.abs(h).reshape(-1, 32).max(axis=1) / 127
            bound += g[t, j] * (np.abs(Wd[e]) @ (np.repeat(step, 32) * (0.5 + 2.0 ** -20)
                                                 + np.abs(h) * 2.0 ** -23))
        diff = np.abs(y8[t] - y16[t])
        assert np.all(diff <= bound + 1e-12), (diff - bound).max()
        assert diff.max() > 0                          # h was quantized


def test_a8_boundary_room_grows_with_eps(orc):
    cfg = S.LayerConfig("a8b", T=2, D=256, E=4, k=2, F=256, qtype="q4_0", x_dtype="f32",
                        y_dtype="f32", seed=37)
    L = S.make_layer(cfg)
    _, ids, g = orc.route(L.x, L.w_router, None, cfg.k)
    out = [orc.layer_a8(L.x, ids, g, L.gate, L.up, L.down, "q4_0", cfg.F, eps=e,
                        want_bound=True) for e in (0.0, 1e-3, 0.5 + 1e-9)]
    ys = [o[0] for o in out]
    bs = [o[1] for o in out]
    for y in ys[1:]:
        np.testing.assert_array_equal(y, ys[0])        # eps only changes the bound
    assert np.all(bs[0] == 0.0)
    assert np.all(bs[1] <= bs[2]) and np.all(bs[1] >= 0)
    # eps past 1/2: every element counts
    assert np.all(bs[2] > 0)
