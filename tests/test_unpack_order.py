"""The K order shared by the weight unpack and the quantised activations on
the mma.sync and tensor-core paths, checked on the CPU.  The GPU expands a
packed word (16 weights; element 16g + 4j + i at bits 8i + 2j) with four
byte-permute lookups in the 4-entry table 0xFFFF0100, one per shift
0, 2, 16, 18 of the word masked to 0x3333.  The quantiser stores each
16-element activation group in the matching order (0,8,1,9, 4,12,5,13,
2,10,3,11, 6,14,7,15).  Restated here in numpy, with the packed words from
the oracle's packer: expanded weights times permuted activations must equal
the plain product in natural order, and the natural-order unpack (shift,
mask, multiply) must give the weights themselves."""

import numpy as np

from oracle import ref

LUT = 0xFFFF0100
PERM = np.array([0, 8, 1, 9, 4, 12, 5, 13, 2, 10, 3, 11, 6, 14, 7, 15])


def byte_perm_table(sel):
    """prmt(LUT, 0, sel) for selectors whose nibbles are 0..3: byte n of the
    result is byte (nibble n) of LUT."""
    out = np.zeros(sel.shape, dtype=np.uint32)
    for n in range(4):
        b = (sel >> (4 * n)) & 0xF
        out |= ((np.uint32(LUT) >> (8 * b).astype(np.uint32)) & 0xFF).astype(np.uint32) << np.uint32(8 * n)
    return out


def expand_permuted(words):
    """[n] uint32 -> [n, 16] int8, bytes in the order of the four lookups."""
    parts = [byte_perm_table((words >> np.uint32(sh)) & np.uint32(0x3333)) for sh in (0, 2, 16, 18)]
    return np.stack(parts, axis=1).view(np.int8).reshape(len(words), 16)


def expand_natural(words):
    """The shift/mask/multiply unpack: lane i of part j is element 4j + i."""
    parts = []
    for j in range(4):
        c = (words >> np.uint32(2 * j)) & np.uint32(0x03030303)
        h = (words >> np.uint32(2 * j + 1)) & np.uint32(0x01010101)
        parts.append((c + h * np.uint32(0xFD)).astype(np.uint32))
    return np.stack(parts, axis=1).view(np.int8).reshape(len(words), 16)


def _case(seed, N=24, K=256):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    packed, gamma = ref.quantize_weights(W)
    q = np.array([[ref.ternary(w, gamma) for w in row] for row in W], dtype=np.int64)
    words = packed.view(np.uint32).reshape(N, K // 16)
    x = rng.integers(-127, 128, K, dtype=np.int64)
    return q, words, x


def test_permuted_unpack_matches_permuted_activations():
    for seed in range(4):
        q, words, x = _case(seed)
        N, G = words.shape
        w8 = expand_permuted(words.ravel()).reshape(N, G, 16).astype(np.int64)
        xp = x.reshape(G, 16)[:, PERM]                  # the quantiser's stored order
        assert np.array_equal((w8 * xp[None]).sum(axis=(1, 2)), q @ x)
        # and element by element: lookup byte p of group g is weight 16g + PERM[p]
        assert np.array_equal(w8, q.reshape(N, G, 16)[:, :, PERM])


def test_natural_unpack_gives_the_weights():
    for seed in range(4):
        q, words, _ = _case(seed + 10)
        N, G = words.shape
        assert np.array_equal(expand_natural(words.ravel()).reshape(N, G * 16), q)


def test_code_three_in_the_byte_permute_unpack():
    """Code 3 is never written.  The byte-permute table reads it as -1; in the
    natural unpack it carries into the next byte lane (c + 0xFD overflows),
    which is the header's "unspecified results" for such input."""
    w = np.array([0xFFFFFFFF], dtype=np.uint32)
    assert np.all(expand_permuted(w) == -1)
    assert not np.all(expand_natural(w) == -1)
