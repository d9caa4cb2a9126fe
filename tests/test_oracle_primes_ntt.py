"""Pins of the oracle's parameter generation and negacyclic NTT.

Primes: every output is prime (trial division), NTT-friendly (= 1 mod 2N),
below 2^bits, in scan order, and no candidate k*2N+1 between two outputs is a
skipped prime.  psi: psi^N = -1 and no smaller x >= 2 has that property.
NTT: the O(N^2) definition, the negacyclic convolution theorem against
schoolbook products, closed forms, and NTT o INTT = id.
"""
import numpy as np
import pytest

from tests import helpers as H


def test_is_prime_matches_trial_division(oracle):
    rng = np.random.default_rng(1)
    xs = list(range(0, 3000)) + [int(v) for v in rng.integers(2**29, 2**32 - 1, size=400)]
    xs += [4294967291, 4294967295, 2147483647, 3215031751, 25326001, 3825123056546413051 % 2**32]
    for x in xs:
        assert oracle.is_prime(x) == H.trial_division_is_prime(x), x


@pytest.mark.parametrize("logN,bits,count", [(10, 30, 8), (12, 30, 6), (16, 31, 28), (17, 31, 45)])
def test_gen_primes_scan(oracle, logN, bits, count):
    pr = [int(v) for v in oracle.gen_primes(logN, bits, count)]
    twoN = 2 << logN
    assert len(pr) == count
    for p in pr:
        assert p < 2**bits and p % twoN == 1 and H.trial_division_is_prime(p)
    # first candidate scanned is floor((2^bits-1)/2N)*2N+1; nothing prime skipped
    k = (2**bits - 1) // twoN
    for p in pr:
        while k * twoN + 1 > p:
            assert not H.trial_division_is_prime(k * twoN + 1), k * twoN + 1
            k -= 1
        assert k * twoN + 1 == p
        k -= 1


def test_chain_assignment(oracle):
    # the first alpha primes found are the special primes, then the L q's
    P = oracle.chain(16, 31, 24, 4)
    allp = oracle.gen_primes(16, 31, 28)
    assert list(P.p) == list(allp[:4]) and list(P.q) == list(allp[4:])
    assert P.dnum == 6
    # every special prime exceeds every ciphertext prime, so P > Q_{D_j}
    assert min(P.p) > max(P.q)


@pytest.mark.parametrize("logN,bits,count", [(10, 30, 3), (12, 30, 2), (16, 31, 2), (17, 31, 2)])
def test_min_psi(oracle, logN, bits, count):
    N = 1 << logN
    for q in oracle.gen_primes(logN, bits, count):
        q = int(q)
        psi = oracle.min_psi(q, logN)
        assert pow(psi, N, q) == q - 1
        # exhaustive: nothing smaller is a primitive 2N-th root
        assert all(pow(x, N, q) != q - 1 for x in range(2, psi))


@pytest.mark.parametrize("logN", [1, 2, 3, 5, 8])
def test_ntt_matches_definition(oracle, logN):
    q = int(oracle.gen_primes(max(logN, 4), 30, 1)[0])  # 2^5 | q-1 covers every logN here
    psi = oracle.min_psi(q, logN)
    a = np.random.default_rng(logN).integers(0, q, size=1 << logN, dtype=np.uint64).astype(np.uint32)
    assert np.array_equal(oracle.ntt_fwd(a, logN, q), H.ntt_by_definition(a, logN, q, psi))


@pytest.mark.parametrize("logN,bits", [(4, 30), (7, 31), (10, 30)])
def test_convolution_theorem(oracle, logN, bits):
    """INTT(NTT(a) * NTT(b)) equals the schoolbook negacyclic product."""
    q = int(oracle.gen_primes(logN, bits, 1)[0])
    g = np.random.default_rng(100 + logN)
    N = 1 << logN
    a = g.integers(0, q, size=N, dtype=np.uint64).astype(np.uint32)
    b = g.integers(0, q, size=N, dtype=np.uint64).astype(np.uint32)
    prod = oracle.ntt_inv(H.mulmod(oracle.ntt_fwd(a, logN, q), oracle.ntt_fwd(b, logN, q), q), logN, q)
    assert np.array_equal(prod, H.negacyclic_schoolbook(a, b, q))


def test_ntt_closed_forms(oracle):
    logN = 12
    N = 1 << logN
    q = int(oracle.gen_primes(logN, 30, 1)[0])
    psi = oracle.min_psi(q, logN)
    one = np.zeros(N, dtype=np.uint32)
    one[0] = 1
    assert np.all(oracle.ntt_fwd(one, logN, q) == 1)
    x = np.zeros(N, dtype=np.uint32)
    x[1] = 1
    want = np.array([pow(psi, 2 * H.bitrev(k, logN) + 1, q) for k in range(N)], dtype=np.uint32)
    assert np.array_equal(oracle.ntt_fwd(x, logN, q), want)
    # X^(N-1): psi^((2brv(k)+1)(N-1))
    x = np.zeros(N, dtype=np.uint32)
    x[N - 1] = 1
    want = np.array([pow(psi, (2 * H.bitrev(k, logN) + 1) * (N - 1), q) for k in range(N)], dtype=np.uint32)
    assert np.array_equal(oracle.ntt_fwd(x, logN, q), want)


@pytest.mark.parametrize("logN,bits", [(12, 30), (16, 31), (17, 31)])
def test_ntt_roundtrip(oracle, logN, bits):
    for q in oracle.gen_primes(logN, bits, 2):
        q = int(q)
        a = np.random.default_rng(q).integers(0, q, size=1 << logN, dtype=np.uint64).astype(np.uint32)
        f = oracle.ntt_fwd(a, logN, q)
        assert np.array_equal(oracle.ntt_inv(f, logN, q), a)
        assert np.array_equal(oracle.ntt_fwd(oracle.ntt_inv(a, logN, q), logN, q), a)
        assert int(f.max()) < q
