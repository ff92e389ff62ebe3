"""The W4A8 GEMV's nibble reorder, checked on the CPU.

A packed word holds eight 4-bit codes, code 2i in the low and code 2i+1 in
the high nibble of byte i.  The GEMV masks the low nibbles (bytes: codes
0, 2, 4, 6) and the high nibbles (codes 1, 3, 5, 7), then builds each A
register of mma.sync from the two with one byte permute: selector 0x5140 for
codes 0..3 and 0x7362 for codes 4..7, so that every lane's codes are in K
order and pair with consecutive activation bytes.  This test restates the
byte-permute rule (each selector nibble picks one of the eight bytes of the
pair {first word, second word}) and checks both selectors on random words."""
import numpy as np

M4 = 0x0F0F0F0F


def byte_perm(x: int, y: int, s: int) -> int:
    pool = [(x >> (8 * i)) & 0xFF for i in range(4)] + [(y >> (8 * i)) & 0xFF for i in range(4)]
    return sum(pool[(s >> (4 * i)) & 7] << (8 * i) for i in range(4))


def test_selectors_put_the_codes_in_k_order():
    rng = np.random.default_rng(15)
    for w in rng.integers(0, 2 ** 32, 2000, dtype=np.uint64):
        w = int(w)
        codes = [(w >> (4 * k)) & 15 for k in range(8)]  # code k: byte k/2, nibble k%2
        lo, hi = w & M4, (w >> 4) & M4
        a0, a2 = byte_perm(lo, hi, 0x5140), byte_perm(lo, hi, 0x7362)
        assert [(a0 >> (8 * i)) & 0xFF for i in range(4)] == codes[0:4]
        assert [(a2 >> (8 * i)) & 0xFF for i in range(4)] == codes[4:8]
    # the plane GEMM's epilogue packs two outputs with the same primitive: the
    # low halves of two words (0x5410) and their high halves (0x7632)
    assert byte_perm(0x11223344, 0x55667788, 0x5410) == 0x77883344
    assert byte_perm(0x11223344, 0x55667788, 0x7632) == 0x55661122
