"""Pins of the oracle's ModUp and ModDown against Python big-integer CRT.

ModUp (approximate FastBConv, Cheon et al. 2018 / Bajard et al. 2016): for a
digit D with coefficient residues x_i, X~ = sum_i [x_i Dhat_i^-1]_{q_i} Dhat_i
satisfies X~ = x (mod Q_D) and 0 <= X~ < |D| Q_D, and ext[t] = NTT_t(X~ mod t);
a one-prime digit converts exactly.  ModDown: out = floor(A/P) - v (mod Q_l)
with v in [0, alpha), v recomputed exactly, and ModDown(P*x) = x exactly.
"""
import numpy as np
import pytest

from tests import helpers as H


def _small(oracle, logN=10, L=5, alpha=2, bits=30):
    pr = oracle.gen_primes(logN, bits, L + alpha)
    return oracle.Params(logN, pr[alpha:], pr[:alpha])


def _rand(P, primes, seed):
    g = np.random.default_rng(seed)
    return np.stack([g.integers(0, int(q), P.N, dtype=np.uint64).astype(np.uint32) for q in primes])


@pytest.mark.parametrize("l", [5, 4, 3, 1])
def test_modup_bigint(oracle, l):
    P = _small(oracle)
    c1 = _rand(P, P.q[:l], 10 + l)
    ext = oracle.modup(P, c1, l)
    beta = -(-l // P.alpha)
    assert ext.shape == (beta, l + P.alpha, P.N)
    x = np.stack([oracle.ntt_inv(c1[i], P.logN, int(P.q[i])) for i in range(l)])
    tprimes = P.level_primes(l)
    for j in range(beta):
        D = list(range(j * P.alpha, min(j * P.alpha + P.alpha, l)))
        QD = H.prod(P.q[i] for i in D)
        Xt = np.zeros(P.N, dtype=object)
        for i in D:
            qi = int(P.q[i])
            Dh = QD // qi
            y = (x[i].astype(object) * pow(Dh % qi, -1, qi)) % qi
            Xt = Xt + y * Dh
        exact = H.crt_lift(x[D], [P.q[i] for i in D])
        u = (Xt - exact)
        assert all(int(v) % QD == 0 for v in u)
        us = np.array([int(v) // QD for v in u])
        assert us.min() >= 0 and us.max() < len(D)
        if len(D) == 1:
            assert us.max() == 0
        for t, qt in enumerate(tprimes):
            if t in D:
                assert np.array_equal(ext[j, t], c1[t])
                continue
            want = np.array([int(v) % qt for v in Xt], dtype=np.uint32)
            assert np.array_equal(oracle.ntt_inv(ext[j, t], P.logN, qt), want), (j, t)


def test_modup_partial_digit_is_exact(oracle):
    # l=5, alpha=2: the last digit holds only q_4, so its conversion is exact
    P = _small(oracle)
    c1 = _rand(P, P.q[:5], 77)
    ext = oracle.modup(P, c1, 5)
    x4 = oracle.ntt_inv(c1[4], P.logN, int(P.q[4]))
    for t, qt in enumerate(P.level_primes(5)):
        if t == 4:
            continue
        want = (x4.astype(np.uint64) % np.uint64(qt)).astype(np.uint32)
        assert np.array_equal(oracle.ntt_inv(ext[2, t], P.logN, qt), want)


@pytest.mark.parametrize("l", [5, 2, 1])
def test_moddown_bigint(oracle, l):
    P = _small(oracle)
    prim = P.level_primes(l)
    acc = np.stack([_rand(P, prim, 200 + l + h) for h in range(2)])
    out = oracle.moddown(P, acc, l)
    Pp = H.prod(P.p)
    Ql = H.prod(P.q[:l])
    for h in range(2):
        coef = np.stack([oracle.ntt_inv(acc[h, t], P.logN, prim[t]) for t in range(l + P.alpha)])
        A = H.crt_lift(coef, prim)
        # exact v from the definition of the fast conversion of the P-residues
        S = np.zeros(P.N, dtype=object)
        for k in range(P.alpha):
            pk = int(P.p[k])
            Ph = Pp // pk
            S = S + ((coef[l + k].astype(object) * pow(Ph % pk, -1, pk)) % pk) * Ph
        v = (S - A % Pp)
        assert all(int(t) % Pp == 0 for t in v)
        v = np.array([int(t) // Pp for t in v])
        assert v.min() >= 0 and v.max() < P.alpha
        want = np.array([(int(a) // Pp - int(vv)) % Ql for a, vv in zip(A, v)], dtype=object)
        got = H.crt_lift(np.stack([oracle.ntt_inv(out[h, i], P.logN, int(P.q[i])) for i in range(l)]),
                         P.q[:l])
        assert all(int(a) == int(b) for a, b in zip(got, want))


def test_moddown_of_P_times_x_is_exact(oracle):
    P = _small(oracle)
    l = 5
    prim = P.level_primes(l)
    Pp = H.prod(P.p)
    x = _rand(P, P.q[:l], 5)
    acc = np.zeros((2, l + P.alpha, P.N), dtype=np.uint32)
    for h in range(2):
        for i in range(l):
            acc[h, i] = H.mulmod(x[i], np.full(P.N, Pp % int(P.q[i]), dtype=np.uint32), int(P.q[i]))
        # P-limbs: P*x = 0 mod p_k (already zero)
    out = oracle.moddown(P, acc, l)
    assert np.array_equal(out[0], x) and np.array_equal(out[1], x)
