"""Writes blocks.txt: hand-packed Standard-family blocks and the values their
closed form gives.

Each block is built from a chosen fp16 scale d (and, for the _1 types, a
chosen fp16 minimum m), each an exactly representable value given both by its
bit pattern and by its exact value, and chosen integer codes; the expected
values are code * d (Q8_0), (code - 8) * d (Q4_0), (code - 16) * d (Q5_0) or
code * d + m (Q4_1, Q5_1), computed here from the chosen integers, never by
decoding the bytes.  The bytes follow the block layouts of the ggml
Standard-family types (FreeToken fork README, "Quant types" table, which names
the types; the layouts are ggml's published ones), little endian:
  Q8_0 = d, then 32 int8 codes;
  Q4_0 = d, then 16 bytes, byte j holding code j in its low nibble and code
         j+16 in its high nibble;
  Q4_1 = d, m, then the 16 nibble bytes as in Q4_0;
  Q5_0 = d, a 32-bit word whose bit i is bit 4 of code i, then the low four
         bits of the codes as Q4_0's 16 bytes;
  Q5_1 = d, m, then the bit-4 word and the 16 nibble bytes as in Q5_0.
K-quants (same table, K-quants row; ggml's published layouts), 256 weights:
  Q4_K = d, dmin, 12 bytes of 6-bit scales sc_j and mins m_j of the eight
         32-weight sub-blocks (j < 4: low six bits of bytes j and j+4;
         j >= 4: the low / high nibble of byte j+4 plus the top two bits of
         bytes j-4 / j), then 128 bytes: weight 64c + l is the low nibble of
         byte 32c + l, weight 64c + 32 + l its high nibble; value
         d * sc_j * q - dmin * m_j;
  Q6_K = 128 bytes ql, 64 bytes qh, 16 int8 scales, d: weight 128h + 32r + l
         has the low four bits in nibble r // 2 of ql[64h + 32(r % 2) + l]
         and the high two in bits 2r, 2r+1 of qh[32h + l]; value
         d * scale[i // 16] * (q - 32).
Run: python tests/golden/make_blocks.py > tests/golden/blocks.txt
"""
from fractions import Fraction

BLOCKS = [
    # name, qtype, d bits, d exact value, codes
    ("q8_unit_ramp", "q8_0", 0x3C00, Fraction(1), [i - 16 for i in range(32)]),
    ("q8_half_extremes", "q8_0", 0x3800, Fraction(1, 2),
     [127, -127, 0, 1, -1, 64, -64, 100] + [(-1) ** i * (3 * i % 120) for i in range(8, 32)]),
    ("q8_subnormal_scale", "q8_0", 0x0001, Fraction(1, 2 ** 24),
     [1, -1, 2, -2] + [0] * 27 + [127]),
    ("q4_half_codes", "q4_0", 0x3800, Fraction(1, 2), [i % 16 for i in range(32)]),
    ("q4_negative_scale", "q4_0", 0xB400, Fraction(-1, 4),
     [15 - i for i in range(16)] + [(7 * i) % 16 for i in range(16, 32)]),
    ("q4_big_scale", "q4_0", 0x5A00, Fraction(192), [0, 15, 8, 7, 9, 1] + [8] * 26),
]

# name, qtype, d bits, d exact, m bits, m exact, codes (the _1 types)
BLOCKS_MIN = [
    ("q4_1_ramp", "q4_1", 0x3800, Fraction(1, 2), 0xC200, Fraction(-3),
     [i % 16 for i in range(32)]),
    ("q4_1_negative_scale", "q4_1", 0xB400, Fraction(-1, 4), 0x3E00, Fraction(3, 2),
     [(5 * i + 3) % 16 for i in range(32)]),
    ("q5_1_scattered_high_bits", "q5_1", 0x3A00, Fraction(3, 4), 0xCA00, Fraction(-12),
     [(11 * i + 5) % 32 for i in range(32)]),
    ("q5_1_subnormal", "q5_1", 0x0001, Fraction(1, 2 ** 24), 0x8001, Fraction(-1, 2 ** 24),
     [31, 0, 1, 30] + [16] * 27 + [15]),
]

BLOCKS_Q5_0 = [
    ("q5_0_full_range", "q5_0", 0x3000, Fraction(1, 8), list(range(32))),
    ("q5_0_scattered_high_bits", "q5_0", 0x4000, Fraction(2), [(7 * i) % 32 for i in range(32)]),
    ("q5_0_only_low_half_high", "q5_0", 0xBC00, Fraction(-1),
     [16 + (i % 16) for i in range(16)] + [i % 16 for i in range(16)]),
]


# name, d bits, d exact, dmin bits, dmin exact, scales[8], mins[8], codes[256]
BLOCKS_Q4K = [
    ("q4_k_mixed_scales", 0x3800, Fraction(1, 2), 0x3400, Fraction(1, 4),
     [1, 2, 3, 63, 17, 40, 5, 33], [0, 1, 62, 7, 48, 3, 21, 63],
     [(7 * i + 3) % 16 for i in range(256)]),
    ("q4_k_negative_scale", 0xBC00, Fraction(-1), 0x4000, Fraction(2),
     [33, 0, 16, 47, 1, 62, 31, 32], [5, 60, 0, 17, 33, 1, 48, 2],
     [(i // 3) % 16 for i in range(256)]),
]

# name, d bits, d exact, scales[16] (int8), codes[256] (0..63)
BLOCKS_Q6K = [
    ("q6_k_signed_scales", 0x3000, Fraction(1, 8),
     [1, -1, 2, -2, 127, -128, 3, 5, -7, 9, 11, -13, 64, -64, 0, 100],
     [(5 * i + 1) % 64 for i in range(256)]),
    ("q6_k_subnormal", 0x0001, Fraction(1, 2 ** 24), [-1] * 16, [i % 64 for i in range(256)]),
]


def pack_q4k(dbits, mbits, sc, mn, codes):
    b = _le16(dbits) + _le16(mbits)
    s12 = [0] * 12
    for j in range(4):
        s12[j] = (sc[j] & 63) | ((sc[j + 4] >> 4) << 6)
        s12[j + 4] = (mn[j] & 63) | ((mn[j + 4] >> 4) << 6)
        s12[j + 8] = (sc[j + 4] & 15) | ((mn[j + 4] & 15) << 4)
    qs = [0] * 128
    for c in range(4):
        for l in range(32):
            qs[32 * c + l] = codes[64 * c + l] | (codes[64 * c + 32 + l] << 4)
    return bytes(b + s12 + qs)


def pack_q6k(dbits, scales, codes):
    ql, qh = [0] * 128, [0] * 64
    for i, q in enumerate(codes):
        h, r, l = i // 128, (i % 128) // 32, i % 32
        ql[64 * h + 32 * (r % 2) + l] |= (q & 15) << (4 * (r // 2))
        qh[32 * h + l] |= (q >> 4) << (2 * r)
    return bytes(ql + qh + [v & 0xFF for v in scales] + _le16(dbits))


def _le16(v):
    return [v & 0xFF, v >> 8]


def _nibbles(codes):
    return [(codes[j] & 0xF) | ((codes[j + 16] & 0xF) << 4) for j in range(16)]


def _high_word(codes):
    w = sum(((c >> 4) & 1) << i for i, c in enumerate(codes))
    return [(w >> (8 * i)) & 0xFF for i in range(4)]


def pack(qtype, dbits, codes, mbits=None):
    b = _le16(dbits)
    if qtype in ("q4_1", "q5_1"):
        b += _le16(mbits)
    if qtype == "q8_0":
        b += [c & 0xFF for c in codes]
    else:
        if qtype in ("q5_0", "q5_1"):
            b += _high_word(codes)
        b += _nibbles(codes)
    return bytes(b)


def main():
    print("# Hand-packed ggml blocks: name qtype hex-bytes then the exact values (32 or 256).")
    print("# Derivation and layout: see make_blocks.py beside this file.")
    def emit(name, qt, raw, vals):
        print(name, qt, raw.hex(), " ".join(repr(float(v)) for v in vals))

    for name, qt, dbits, d, codes in BLOCKS:
        assert len(codes) == 32
        if qt == "q8_0":
            vals = [c * d for c in codes]
        else:
            vals = [(c - 8) * d for c in codes]
        emit(name, qt, pack(qt, dbits, codes), vals)
    for name, qt, dbits, d, codes in BLOCKS_Q5_0:
        assert len(codes) == 32 and all(0 <= c < 32 for c in codes)
        emit(name, qt, pack(qt, dbits, codes), [(c - 16) * d for c in codes])
    for name, qt, dbits, d, mbits, m, codes in BLOCKS_MIN:
        top = 16 if qt == "q4_1" else 32
        assert len(codes) == 32 and all(0 <= c < top for c in codes)
        emit(name, qt, pack(qt, dbits, codes, mbits), [c * d + m for c in codes])
    for name, dbits, d, mbits, dmin, sc, mn, codes in BLOCKS_Q4K:
        assert len(codes) == 256 and all(0 <= c < 16 for c in codes)
        assert all(0 <= v < 64 for v in sc + mn)
        vals = [d * sc[i // 32] * codes[i] - dmin * mn[i // 32] for i in range(256)]
        emit(name, "q4_k", pack_q4k(dbits, mbits, sc, mn, codes), vals)
    for name, dbits, d, scales, codes in BLOCKS_Q6K:
        assert len(codes) == 256 and all(0 <= c < 64 for c in codes)
        assert all(-128 <= v < 128 for v in scales)
        vals = [d * scales[i // 16] * (codes[i] - 32) for i in range(256)]
        emit(name, "q6_k", pack_q6k(dbits, scales, codes), vals)


if __name__ == "__main__":
    main()
