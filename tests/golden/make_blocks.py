"""Writes blocks.txt: hand-packed Q8_0 / Q4_0 blocks and the values their
closed form gives.

Each block is built from a chosen fp16 scale (an exactly representable value,
given by its bit pattern) and chosen integer codes; the expected values are
code * d (Q8_0) or (code - 8) * d (Q4_0), computed here from the chosen
integers, never by decoding the bytes.  The bytes follow the block layouts of
the ggml Standard-family types (FreeToken fork README, "Quant types" table):
Q8_0 = fp16 d (little endian) then 32 int8 codes; Q4_0 = fp16 d then 16 bytes,
byte j holding code j in its low nibble and code j+16 in its high nibble.
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


def pack(qtype, dbits, codes):
    b = [dbits & 0xFF, dbits >> 8]
    if qtype == "q8_0":
        b += [c & 0xFF for c in codes]
    else:
        b += [codes[j] | (codes[j + 16] << 4) for j in range(16)]
    return bytes(b)


def main():
    print("# Hand-packed ggml blocks: name qtype hex-bytes then 32 exact values.")
    print("# Derivation and layout: see make_blocks.py beside this file.")
    for name, qt, dbits, d, codes in BLOCKS:
        assert len(codes) == 32
        if qt == "q8_0":
            vals = [c * d for c in codes]
        else:
            vals = [(c - 8) * d for c in codes]
        print(name, qt, pack(qt, dbits, codes).hex(), " ".join(repr(float(v)) for v in vals))


if __name__ == "__main__":
    main()
