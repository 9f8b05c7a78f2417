"""Philox-4x64-10 counter-based generator, written from its published definition.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import this module;
only tests/, the package's smoke check and the bench's CPU-baseline leg call it.

Source of the definition: J. Salmon, M. Moraes, R. Dror, D. Shaw, "Parallel
Random Numbers: As Easy as 1, 2, 3", SC'11 -- the Philox-4x64 round (two
64x64->128-bit multiplies whose high halves are XORed with the other two
counter words and the key), the Weyl key schedule, 10 rounds.

How the canvas uses it (the pages fix only that the canvas starts as uniform
random token ids and that uncertain positions are re-randomised; see
"DiffusionGemma解析", section 整片并行去噪, and "谷歌DiffusionGemma", section
工作原理): key = (seed_b, 0), counter = (position, step, canvas, 0), word 0 of
the output block; the token id is the top 32 bits of that word scaled to the
vocabulary with a multiply-shift.

Everything here uses plain Python integers so each operation can be read off
against the paper.
"""

MASK64 = (1 << 64) - 1

# Multipliers and Weyl increments of Philox-4x64 (Salmon et al., table of constants).
PHILOX_M0 = 0xD2E7470EE14C6C93
PHILOX_M1 = 0xCA5A826395121157
PHILOX_W0 = 0x9E3779B97F4A7C15
PHILOX_W1 = 0xBB67AE8584CAA73B
PHILOX_ROUNDS = 10


def _mulhilo(a, b):
    prod = (a & MASK64) * (b & MASK64)
    return (prod >> 64) & MASK64, prod & MASK64


def philox4x64_10(counter, key):
    """One Philox-4x64-10 block: 4 x 64-bit counter words, 2 x 64-bit key words
    -> 4 x 64-bit output words."""
    x0, x1, x2, x3 = (int(c) & MASK64 for c in counter)
    k0, k1 = (int(k) & MASK64 for k in key)
    for r in range(PHILOX_ROUNDS):
        if r > 0:  # key schedule: bump the key before every round but the first
            k0 = (k0 + PHILOX_W0) & MASK64
            k1 = (k1 + PHILOX_W1) & MASK64
        hi0, lo0 = _mulhilo(PHILOX_M0, x0)
        hi1, lo1 = _mulhilo(PHILOX_M1, x2)
        x0, x1, x2, x3 = hi1 ^ x1 ^ k0, lo1, hi0 ^ x3 ^ k1, lo0
    return x0, x1, x2, x3


def token_from_word(word0, vocab):
    """Map the top 32 bits of a 64-bit word onto [0, vocab) by multiply-shift.
    Exactly uniform when vocab is a power of two."""
    return ((int(word0) >> 32) * int(vocab)) >> 32


def canvas_draw(seed, step, position, canvas, vocab):
    """Token id drawn for (seed, step, position, canvas). step 0 is the initial
    canvas; step t+1 is the re-noise after denoise step t."""
    w = philox4x64_10((position, step, canvas, 0), (seed, 0))
    return token_from_word(w[0], vocab)
