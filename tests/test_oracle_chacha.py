"""Pins of the oracle's ChaCha core and of the key-regeneration mapping.

The pages name the expander only ("ChaCha12 counter-mode expander", arxivlens
summary of the Perseus paper, "Methodology"; Perseus README, "What's inside").
The round function is pinned to the `cryptography` package's ChaCha20
(an independent implementation); ChaCha12 is the same permutation stopped
after 6 double rounds, pinned by composition; the spec-v1 word layout and
the (hi*2^32 + lo) mod q mapping are pinned by running the same expander
with 20 rounds against `cryptography`'s keystream.
"""
import struct

import numpy as np
import pytest
from cryptography.hazmat.primitives.ciphers import Cipher, algorithms

SIGMA = [0x61707865, 0x3320646E, 0x79622D32, 0x6B206574]


def _keystream20(key: bytes, words12_15, nbytes: int) -> bytes:
    nonce = struct.pack("<4I", *words12_15)
    enc = Cipher(algorithms.ChaCha20(key, nonce), mode=None).encryptor()
    return enc.update(b"\0" * nbytes)


def _state(key: bytes, w12, w13, w14, w15):
    return SIGMA + list(struct.unpack("<8I", key)) + [w12, w13, w14, w15]


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_chacha20_block_matches_cryptography(oracle, seed):
    g = np.random.default_rng(seed)
    key = g.integers(0, 256, 32, dtype=np.uint8).tobytes()
    w = [int(v) for v in g.integers(0, 2**32, 4, dtype=np.uint64)]
    out = oracle.chacha_block(_state(key, *w), rounds=20)
    assert out.astype("<u4").tobytes() == _keystream20(key, w, 64)


def test_counter_mode_continuation(oracle):
    key = bytes(range(32))
    ks = _keystream20(key, [0, 7, 3, 0x61], 128)
    b1 = oracle.chacha_block(_state(key, 1, 7, 3, 0x61), rounds=20)
    assert b1.astype("<u4").tobytes() == ks[64:]


def test_chacha12_is_six_double_rounds(oracle):
    """permute(10) = permute(4) o permute(6); ChaCha20 = permute(10) + input
    (pinned above), so permute(6) is the first 6 double rounds of the pinned
    permutation, and ChaCha12 = permute(6) + input."""
    key = bytes(range(1, 33))
    st = np.array(_state(key, 5, 9, 2, 0x61), dtype=np.uint32)
    p6 = oracle.chacha_permute(st, 6)
    p10 = oracle.chacha_permute(st, 10)
    assert np.array_equal(oracle.chacha_permute(p6, 4), p10)
    assert np.array_equal((p10 + st).astype(np.uint32), oracle.chacha_block(st, 20))
    assert np.array_equal((p6 + st).astype(np.uint32), oracle.chacha_block(st, 12))
    assert not np.array_equal(oracle.chacha_block(st, 12), oracle.chacha_block(st, 20))


@pytest.mark.parametrize("j,g,logN", [(0, 0, 6), (3, 17, 8), (5, 27, 7)])
def test_expand_mapping_layout(oracle, j, g, logN):
    """Spec v1: state words 12..15 = (block counter, global prime index,
    digit, 0x61); coefficient k takes words 2(k%8), 2(k%8)+1 of block k/8 as
    lo, hi, and a = (hi*2^32 + lo) mod q."""
    P = oracle.chain(16, 31, 24, 4)
    q = P.prime(g)
    seed = bytes((7 * i + 3) % 256 for i in range(32))
    N = 1 << logN
    want = []
    for b in range(N // 8):
        ks = np.frombuffer(_keystream20(seed, [b, g, j, 0x61], 64), dtype="<u4")
        for w in range(8):
            want.append(((int(ks[2 * w + 1]) << 32) | int(ks[2 * w])) % q)
    got = oracle.expand_a(seed, j, g, q, logN, rounds=20)
    assert [int(v) for v in got] == want


def test_expand12_uniform_chi2(oracle):
    P = oracle.chain(16, 31, 24, 4)
    q = P.prime(3)
    a = oracle.expand_a(bytes(32), 1, 3, q, 16).astype(np.float64)
    assert a.max() < q
    bins = np.bincount((a * 64 / q).astype(np.int64), minlength=64)
    exp = len(a) / 64
    chi2 = float(((bins - exp) ** 2 / exp).sum())
    assert chi2 < 120.0, chi2  # 63 dof; p < 1e-5 at 120


def test_expand12_streams_distinct(oracle):
    P = oracle.chain(12, 30, 4, 2)
    s = bytes(range(32))
    a00 = oracle.expand_a(s, 0, 0, P.prime(0), 12)
    a10 = oracle.expand_a(s, 1, 0, P.prime(0), 12)
    a01 = oracle.expand_a(s, 0, 1, P.prime(0), 12)
    assert not np.array_equal(a00, a10) and not np.array_equal(a00, a01)
