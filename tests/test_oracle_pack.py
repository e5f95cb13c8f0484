"""Pins for the oracle's packed layout and dequantization.

The layout is our own (the pages name only a ".pt" checkpoint); it is fixed in
include/awq.h and the hand-derived words in tests/golden/packed_words.txt pin
it. Dequantization is pinned to numpy's own fp16 rounding of the exact
product (q - z) s.
"""
import numpy as np
import pytest

import oracle
from golden_io import packed_words

G = 128


def test_single_nibbles_land_on_hand_derived_words():
    for N, K, n, k, qv, widx, wval, g in packed_words():
        q = np.zeros((N, K), np.uint8)
        q[n, k] = qv
        z = np.zeros((N, K // g), np.uint8)
        s = np.zeros((N, K // g), np.float16)
        qw, _, _ = oracle.pack(q, z, s, g)
        flat = qw.reshape(-1)
        nz = np.flatnonzero(flat)
        assert list(nz) == [widx], (n, k, nz)
        assert flat[widx] == wval, (n, k, hex(flat[widx]))


def test_whole_word_interleave():
    # k = 0..7 of row 0 hold q = 0..7: even k go to the low half-word, odd k
    # to the high half-word, each pair (2j, 2j+1) four bits further up.
    q = np.zeros((16, G), np.uint8)
    q[0, :8] = np.arange(8)
    qw, _, _ = oracle.pack(q, np.zeros((16, 1), np.uint8), np.zeros((16, 1), np.float16), G)
    assert qw.reshape(-1)[0] == 0x75316420
    # the pair k = (2j, 2j+1) is (word >> 4j) & 0x000F000F as two 16-bit lanes
    w = int(qw.reshape(-1)[0])
    for j in range(4):
        pair = (w >> (4 * j)) & 0x000F000F
        assert (pair & 0xFFFF, pair >> 16) == (2 * j, 2 * j + 1)


def test_scale_and_zero_layout():
    N, K = 16, 2 * G
    q = np.zeros((N, K), np.uint8)
    z = np.zeros((N, K // G), np.uint8)
    s = np.zeros((N, K // G), np.float16)
    z[3, 1] = 0xB          # odd n -> high nibble of byte g*(N/2) + n/2 = 8 + 1
    z[6, 0] = 0x4          # even n -> low nibble of byte 0*8 + 3
    s[5, 1] = 1.5          # scales are [K/G][N]: element 1*16 + 5
    _, sc, ze = oracle.pack(q, z, s, G)
    assert ze.reshape(-1)[9] == 0xB0 and ze.reshape(-1)[3] == 0x04
    assert np.count_nonzero(ze) == 2
    assert sc.reshape(-1)[21] == np.float16(1.5) and np.count_nonzero(sc) == 1


@pytest.mark.parametrize("G", [128, 64, 32])
def test_pack_unpack_round_trips(G):
    rng = np.random.default_rng(11)
    for N, K in [(16, 128), (48, 384), (64, 1024)]:
        q = rng.integers(0, 16, (N, K)).astype(np.uint8)
        z = rng.integers(0, 16, (N, K // G)).astype(np.uint8)
        s = rng.integers(0, 0x7C00, (N, K // G)).astype(np.uint16).view(np.float16)
        qw, sc, ze = oracle.pack(q, z, s, G)
        q2, z2, s2 = oracle.unpack(qw, sc, ze, N, K, G)
        assert (q2 == q).all() and (z2 == z).all() and (s2.view(np.uint16) == s.view(np.uint16)).all()
        # and the other direction: random packed buffers survive unpack + pack
        qw_r = rng.integers(0, 2 ** 32, qw.shape, dtype=np.uint64).astype(np.uint32)
        ze_r = rng.integers(0, 256, ze.shape).astype(np.uint8)
        q3, z3, s3 = oracle.unpack(qw_r, sc, ze_r, N, K, G)
        qw2, sc2, ze2 = oracle.pack(q3, z3, s3, G)
        assert (qw2 == qw_r).all() and (ze2 == ze_r).all() and (sc2.view(np.uint16) == sc.view(np.uint16)).all()


@pytest.mark.parametrize("G", [64, 32])
def test_words_of_one_group_size_hold_whole_groups(G):
    """G = 64, 32: the four words 4t .. 4t+3 a GPU lane reads hold one 8-input
    piece of every group of the k-block, and the words with the same j (word
    index mod 4) hold whole groups, group j / (G / 32); within a word the eight
    inputs stay consecutive."""
    N, K = 16, 128
    J = G // 32
    q = np.zeros((N, K), np.uint8)
    q[:, :] = (np.arange(K) // G + 1)[None, :]          # group index + 1
    qw, _, _ = oracle.pack(q, np.zeros((N, K // G), np.uint8), np.zeros((N, K // G), np.float16), G)
    words = qw.reshape(-1)[:16]                          # row 0 of the only block
    for w, word in enumerate(words):
        nib = [(int(word) >> sh) & 0xF for sh in (0, 16, 4, 20, 8, 24, 12, 28)]  # i = 0..7
        assert len(set(nib)) == 1 and nib[0] == (w % 4) // J + 1, (w, hex(int(word)))
    # consecutive inputs: q = k % 8 shows the order inside every word
    q[:, :] = (np.arange(K) % 8)[None, :]
    qw, _, _ = oracle.pack(q, np.zeros((N, K // G), np.uint8), np.zeros((N, K // G), np.float16), G)
    assert (qw.reshape(-1)[:16] == 0x75316420).all()


@pytest.mark.parametrize("G", [128, 64, 32])
def test_dequant_is_numpy_rounding_of_the_exact_product(G):
    rng = np.random.default_rng(5)
    N, K = 32, 4 * G
    q = rng.integers(0, 16, (N, K)).astype(np.uint8)
    z = rng.integers(0, 16, (N, K // G)).astype(np.uint8)
    # scales over the whole finite fp16 range, subnormals included
    s = rng.integers(1, 0x7C00, (N, K // G)).astype(np.uint16).view(np.float16)
    wh = oracle.dequant(q, z, s, G)
    exact = (q.astype(np.float64) - np.repeat(z, G, axis=1)) * np.repeat(s.astype(np.float64), G, axis=1)
    with np.errstate(over="ignore"):
        ref = exact.astype(np.float16)
    assert (wh.view(np.uint16) == ref.view(np.uint16)).all()
