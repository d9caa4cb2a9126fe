"""Pins of the oracle's key generation and full key switch.

Keygen identity: b_j + a_j*s - [P]_q * g_j * s' recomputed equals e_j exactly
(coefficient form).  Automorphism: s(X^g) by brute-force substitution.

Key switch (hybrid key switching, Han-Ki 2020): decryption under the true
secret after switching s' -> s matches decryption before, within

    B = sum_j |D_j| Q_{D_j} ||e_j||_1 / P + (1 + alpha)(1 + ||s||_1).

Derivation.  Let A_h be the integer lift of acc_h over Q_l P.  With d~_j the
ModUp value of digit j (0 <= d~_j < |D_j| Q_{D_j}) and b_j + a_j s = e_j +
P G_j s' (G_j = 1 mod the digit's primes, 0 mod the other q's),
A_b + A_a s = P c1 s' + E (mod Q_l P), E = sum_j d~_j e_j, because
sum_j d~_j G_j = c1 (mod Q_l).  ModDown gives out_h = (A_h - r_h)/P - v_h with
r_h = A_h mod P and 0 <= v_h < alpha.  Hence
(c0' + c1' s) - (c0 + c1 s') = E/P - (r_b + r_a s)/P - v_b - v_a s (mod Q_l),
and |E/P| <= sum_j ||d~_j||_inf ||e_j||_1 / P, |r_b/P| < 1, |r_a s/P| < ||s||_1,
|v_b| < alpha, |v_a s| <= alpha ||s||_1.  A wrong key breaks the bound (teeth),
and every tested bound is below Q_l/2.
"""
import numpy as np
import pytest

from key_switching_b200 import synth
from tests import helpers as H


def _setup(oracle, logN, L, alpha, bits, key="square", hw=None, seed=0, r=1):
    pr = oracle.gen_primes(logN, bits, L + alpha)
    P = oracle.Params(logN, pr[alpha:], pr[:alpha])
    s = synth.ternary_secret(P.N, seed, hw)
    if key == "square":
        sp = oracle.negacyclic_mul(s, s, logN)
    else:
        sp = oracle.automorph(s, logN, oracle.galois_elt(r, logN))
    e = synth.gaussian_errors(P.dnum, P.N, seed)
    kseed = synth.chacha_seed(seed, r)
    b = oracle.ksk_gen(P, s, sp, e, kseed)
    return P, s, sp, e, kseed, b


def test_automorph_bruteforce(oracle):
    logN = 5
    N = 1 << logN
    s = np.random.default_rng(3).integers(-5, 6, N).astype(np.int64)
    for r in [1, 2, 7]:
        g = oracle.galois_elt(r, logN)
        want = [0] * N
        for n in range(N):
            e = n * g
            sign = -1 if (e // N) % 2 else 1   # X^N = -1
            want[e % N] += sign * int(s[n])
        assert list(oracle.automorph(s, logN, g)) == want


def test_negacyclic_mul_small(oracle):
    a = np.array([1, 2, 0, -1], dtype=np.int64)
    b = np.array([0, 1, 0, 0], dtype=np.int64)  # times X
    assert list(oracle.negacyclic_mul(a, b, 2)) == [1, 1, 2, 0]


@pytest.mark.parametrize("logN,L,alpha,bits,key", [(10, 5, 2, 30, "square"), (12, 4, 2, 30, "square"),
                                                   (11, 6, 3, 31, "rot")])
def test_keygen_identity(oracle, logN, L, alpha, bits, key):
    P, s, sp, e, kseed, b = _setup(oracle, logN, L, alpha, bits, key)
    Pp = H.prod(P.p)
    for j in range(P.dnum):
        for g in range(P.L + P.alpha):
            q = P.prime(g)
            a = oracle.expand_a(kseed, j, g, q, logN)
            sh = oracle.ntt_fwd(H.reduce_signed(s, q), logN, q)
            v = H.addmod(b[j, g], H.mulmod(a, sh, q), q)
            if g < P.L and j * alpha <= g < j * alpha + alpha:
                sph = oracle.ntt_fwd(H.reduce_signed(sp, q), logN, q)
                v = H.submod(v, H.mulmod(np.full(P.N, Pp % q, dtype=np.uint32), sph, q), q)
            assert np.array_equal(oracle.ntt_inv(v, logN, q), H.reduce_signed(e[j], q)), (j, g)


def _decrypt_error(oracle, P, l, s, sp, e, kseed, b, c0, c1, a=None):
    c0o, c1o = oracle.keyswitch(P, c0, c1, l, kseed, b, a)
    diffs = []
    for i in range(l):
        q = int(P.q[i])
        sh = oracle.ntt_fwd(H.reduce_signed(s, q), P.logN, q)
        sph = oracle.ntt_fwd(H.reduce_signed(sp, q), P.logN, q)
        after = H.addmod(c0o[i], H.mulmod(c1o[i], sh, q), q)
        before = H.addmod(c0[i], H.mulmod(c1[i], sph, q), q)
        diffs.append(oracle.ntt_inv(H.submod(after, before, q), P.logN, q))
    Ql = H.prod(P.q[:l])
    err = H.centered(H.crt_lift(np.stack(diffs), P.q[:l]), Ql)
    return max(abs(int(v)) for v in err), Ql


def _bound(P, l, s, e):
    Pp = H.prod(P.p)
    beta = -(-l // P.alpha)
    t = 0
    for j in range(beta):
        D = list(range(j * P.alpha, min(j * P.alpha + P.alpha, l)))
        t += len(D) * H.prod(P.q[i] for i in D) * int(np.abs(e[j]).sum())
    return t // Pp + 1 + (1 + P.alpha) * (1 + int(np.abs(s).sum()))


@pytest.mark.parametrize("logN,L,alpha,bits,key,hw", [
    (12, 4, 2, 30, "square", None),   # the N=2^12 relinearisation workload's shape
    (10, 5, 2, 30, "square", None),   # partial last digit
    (11, 7, 3, 31, "rot", 64),        # 31-bit primes, alpha=3, partial digit
])
def test_decrypt_after_keyswitch(oracle, logN, L, alpha, bits, key, hw):
    P, s, sp, e, kseed, b = _setup(oracle, logN, L, alpha, bits, key, hw)
    for l in sorted({L, L - 1, 1, max(1, alpha + 1)}, reverse=True):
        c0 = np.stack([synth.uniform_residues([q], P.N, 9, l, i)[0] for i, q in enumerate(P.q[:l])])
        c1 = np.stack([synth.uniform_residues([q], P.N, 8, l, i)[0] for i, q in enumerate(P.q[:l])])
        err, Ql = _decrypt_error(oracle, P, l, s, sp, e, kseed, b, c0, c1)
        bound = _bound(P, l, s, e)
        assert bound < Ql // 2
        assert err <= bound, (l, err, bound)


def test_stored_a_equals_regenerated(oracle):
    P, s, sp, e, kseed, b = _setup(oracle, 10, 5, 2, 30)
    l = 5
    a = np.zeros_like(b)
    for j in range(P.dnum):
        for g in range(P.L + P.alpha):
            a[j, g] = oracle.expand_a(kseed, j, g, P.prime(g), P.logN)
    c0 = synth.uniform_residues(P.q[:l], P.N, 1)
    c1 = synth.uniform_residues(P.q[:l], P.N, 2)
    r1 = oracle.keyswitch(P, c0, c1, l, kseed, b)
    r2 = oracle.keyswitch(P, c0, c1, l, kseed, b, a)
    assert np.array_equal(r1[0], r2[0]) and np.array_equal(r1[1], r2[1])


def test_wrong_key_fails(oracle):
    """Teeth: a key for a different s' gives an error far above the bound."""
    P, s, sp, e, kseed, b = _setup(oracle, 10, 5, 2, 30)
    l = 5
    c0 = synth.uniform_residues(P.q[:l], P.N, 1)
    c1 = synth.uniform_residues(P.q[:l], P.N, 2)
    sp_wrong = sp.copy()
    sp_wrong[0] += 1
    err, Ql = _decrypt_error(oracle, P, l, s, sp_wrong, e, kseed, b, c0, c1)
    assert err > 1000 * _bound(P, l, s, e)


@pytest.mark.slow
def test_decrypt_rotation_n16(oracle):
    """The N=2^16, L=24, alpha=4 rotation workload at the top level."""
    P, s, sp, e, kseed, b = _setup(oracle, 16, 24, 4, 31, "rot", synth.HAMMING_WEIGHT)
    l = 24
    c0 = synth.uniform_residues(P.q[:l], P.N, 1)
    c1 = synth.uniform_residues(P.q[:l], P.N, 2)
    err, Ql = _decrypt_error(oracle, P, l, s, sp, e, kseed, b, c0, c1)
    bound = _bound(P, l, s, e)
    assert err <= bound < Ql // 2
