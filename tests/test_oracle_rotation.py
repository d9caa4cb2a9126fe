"""Pins of the oracle's rotation and relinearisation paths.

NTT-domain automorphism: checked against the coefficient-domain substitution
s(X) -> s(X^g) (itself pinned by brute force) through the pinned forward NTT,
and against the group law sigma_h(sigma_g(a)) = sigma_{gh}(a).

Rotation (automorphism, then hybrid key switching with a key for
s(X^g) -> s): decryption under s after the rotation matches
c0(X^g) + c1(X^g) s(X^g) within the key-switching bound B of
test_oracle_keyswitch (the automorphism permutes coefficients, so the lifted
digits and their bounds are unchanged).  Hoisted rotations (ModUp of c1 once,
automorphism applied to the extended limbs) decrypt within the same bound, and
with g = 1 equal the plain key switch exactly.

Relinearisation: the tensor is the slot-wise product (pinned against the
negacyclic schoolbook product through the NTT), and after switching d2 with a
key for s^2 -> s, c0' + c1' s matches d0 + d1 s + d2 s^2 within B.
"""
import numpy as np
import pytest

from key_switching_b200 import synth
from tests import helpers as H
from tests.test_oracle_keyswitch import _bound, _setup


def _ntt_of_int(oracle, a, logN, q):
    return oracle.ntt_fwd(H.reduce_signed(a, q), logN, q)


@pytest.mark.parametrize("logN", [4, 8, 10])
def test_automorph_ntt_matches_coefficient_substitution(oracle, logN):
    N = 1 << logN
    q = int(oracle.gen_primes(logN, 30, 1)[0])
    a = np.random.default_rng(logN).integers(-1000, 1001, N).astype(np.int64)
    for g in sorted({1, 3, 5, 2 * N - 1, oracle.galois_elt(7, logN), oracle.galois_elt(N // 4 + 1, logN)}):
        want = _ntt_of_int(oracle, oracle.automorph(a, logN, g), logN, q)
        got = oracle.automorph_ntt(_ntt_of_int(oracle, a, logN, q), logN, g)
        assert np.array_equal(got, want), g


def test_automorph_ntt_group_law(oracle):
    logN = 9
    N = 1 << logN
    x = np.random.default_rng(1).integers(0, 2**30, N).astype(np.uint32)
    assert np.array_equal(oracle.automorph_ntt(x, logN, 1), x)
    for g, h in [(5, 25), (3, 2 * N - 1), (oracle.galois_elt(11, logN), 7)]:
        two = oracle.automorph_ntt(oracle.automorph_ntt(x, logN, g), logN, h)
        assert np.array_equal(two, oracle.automorph_ntt(x, logN, g * h % (2 * N)))


def _rot_error(oracle, P, l, s, g, c0, c1, c0o, c1o):
    """max |(c0o + c1o s) - (c0(X^g) + c1(X^g) s(X^g))| over Q_l (centred)."""
    sg = oracle.automorph(s, P.logN, g)
    diffs = []
    for i in range(l):
        q = int(P.q[i])
        sh = _ntt_of_int(oracle, s, P.logN, q)
        sgh = _ntt_of_int(oracle, sg, P.logN, q)
        after = H.addmod(c0o[i], H.mulmod(c1o[i], sh, q), q)
        r0 = oracle.automorph_ntt(c0[i], P.logN, g)
        r1 = oracle.automorph_ntt(c1[i], P.logN, g)
        before = H.addmod(r0, H.mulmod(r1, sgh, q), q)
        diffs.append(oracle.ntt_inv(H.submod(after, before, q), P.logN, q))
    Ql = H.prod(P.q[:l])
    err = H.centered(H.crt_lift(np.stack(diffs), P.q[:l]), Ql)
    return max(abs(int(v)) for v in err), Ql


def _ct(P, l, seed):
    c0 = np.stack([synth.uniform_residues([q], P.N, seed, l, i)[0] for i, q in enumerate(P.q[:l])])
    c1 = np.stack([synth.uniform_residues([q], P.N, seed + 1, l, i)[0] for i, q in enumerate(P.q[:l])])
    return c0, c1


@pytest.mark.parametrize("logN,L,alpha,bits,r", [(10, 5, 2, 30, 1), (11, 7, 3, 31, 5), (10, 4, 2, 30, -1)])
def test_decrypt_after_rotation(oracle, logN, L, alpha, bits, r):
    rr = r if r >= 0 else (1 << (logN - 1)) - 1  # -1: the last slot rotation
    P, s, sp, e, kseed, b = _setup(oracle, logN, L, alpha, bits, "rot", r=rr)
    g = oracle.galois_elt(rr, logN)
    for l in sorted({L, 1, alpha + 1}, reverse=True):
        c0, c1 = _ct(P, l, 20)
        c0o, c1o = oracle.rotate(P, c0, c1, l, g, kseed, b)
        err, Ql = _rot_error(oracle, P, l, s, g, c0, c1, c0o, c1o)
        bound = _bound(P, l, s, e)
        assert bound < Ql // 2
        assert err <= bound, (l, err, bound)


def test_rotation_with_wrong_galois_element_fails(oracle):
    """Teeth: the key for g does not switch an automorphism by another element."""
    P, s, sp, e, kseed, b = _setup(oracle, 10, 5, 2, 30, "rot", r=3)
    g = oracle.galois_elt(3, 10)
    c0, c1 = _ct(P, 5, 30)
    c0o, c1o = oracle.rotate(P, c0, c1, 5, oracle.galois_elt(4, 10), kseed, b)
    err, _ = _rot_error(oracle, P, 5, s, oracle.galois_elt(4, 10), c0, c1, c0o, c1o)
    assert err > 1000 * _bound(P, 5, s, e)
    c0o, c1o = oracle.rotate(P, c0, c1, 5, g, kseed, b)
    assert _rot_error(oracle, P, 5, s, g, c0, c1, c0o, c1o)[0] <= _bound(P, 5, s, e)


def test_hoisted_rotations(oracle):
    logN, L, alpha = 10, 6, 2
    rs = [1, 2, 7]
    keys = [_setup(oracle, logN, L, alpha, 30, "rot", seed=0, r=r) for r in rs]
    P, s, _, e, _, _ = keys[0]
    gs = [oracle.galois_elt(r, logN) for r in rs]
    for l in (L, 3):
        c0, c1 = _ct(P, l, 40)
        outs = oracle.rotate_hoisted(P, c0, c1, l, gs, [k[4] for k in keys], [k[5] for k in keys])
        for g, (c0o, c1o) in zip(gs, outs):
            err, Ql = _rot_error(oracle, P, l, s, g, c0, c1, c0o, c1o)
            assert err <= _bound(P, l, s, e) < Ql // 2, (l, g, err)


def test_hoisted_identity_is_keyswitch(oracle):
    P, s, sp, e, kseed, b = _setup(oracle, 10, 5, 2, 30, "square")
    c0, c1 = _ct(P, 5, 50)
    (h0, h1), = oracle.rotate_hoisted(P, c0, c1, 5, [1], [kseed], [b])
    k0, k1 = oracle.keyswitch(P, c0, c1, 5, kseed, b)
    assert np.array_equal(h0, k0) and np.array_equal(h1, k1)
    r0, r1 = oracle.rotate(P, c0, c1, 5, 1, kseed, b)
    assert np.array_equal(r0, k0) and np.array_equal(r1, k1)


def test_tensor_is_ring_product(oracle):
    logN = 8
    N = 1 << logN
    pr = oracle.gen_primes(logN, 30, 3)
    P = oracle.Params(logN, pr[1:], pr[:1])
    rng = np.random.default_rng(5)
    xi = [rng.integers(-50, 51, N).astype(np.int64) for _ in range(4)]
    q = int(P.q[0])
    x0, x1, y0, y1 = [_ntt_of_int(oracle, v, logN, q)[None, :] for v in xi]
    d0, d1, d2 = oracle.tensor(P, x0, x1, y0, y1, 1)
    m = oracle.negacyclic_mul
    assert np.array_equal(d0[0], _ntt_of_int(oracle, m(xi[0], xi[2], logN), logN, q))
    assert np.array_equal(d1[0], _ntt_of_int(oracle, m(xi[0], xi[3], logN) + m(xi[1], xi[2], logN), logN, q))
    assert np.array_equal(d2[0], _ntt_of_int(oracle, m(xi[1], xi[3], logN), logN, q))


@pytest.mark.parametrize("logN,L,alpha,bits", [(12, 4, 2, 30), (10, 5, 2, 30)])
def test_decrypt_after_relinearisation(oracle, logN, L, alpha, bits):
    P, s, s2, e, kseed, b = _setup(oracle, logN, L, alpha, bits, "square")
    for l in (L, 2):
        x0, x1 = _ct(P, l, 60)
        y0, y1 = _ct(P, l, 70)
        c0o, c1o = oracle.relinearize(P, x0, x1, y0, y1, l, kseed, b)
        d0, d1, d2 = oracle.tensor(P, x0, x1, y0, y1, l)
        diffs = []
        for i in range(l):
            q = int(P.q[i])
            sh = _ntt_of_int(oracle, s, logN, q)
            s2h = _ntt_of_int(oracle, s2, logN, q)
            after = H.addmod(c0o[i], H.mulmod(c1o[i], sh, q), q)
            before = H.addmod(H.addmod(d0[i], H.mulmod(d1[i], sh, q), q), H.mulmod(d2[i], s2h, q), q)
            diffs.append(oracle.ntt_inv(H.submod(after, before, q), logN, q))
        Ql = H.prod(P.q[:l])
        err = max(abs(int(v)) for v in H.centered(H.crt_lift(np.stack(diffs), P.q[:l]), Ql))
        assert err <= _bound(P, l, s, e) < Ql // 2, (l, err)


@pytest.mark.parametrize("logN", [10, 12, 16, 17])
def test_automorphism_maps_row_blocks_to_row_blocks(oracle, logN):
    """The property the GPU rotation kernels are built on, derived from the
    oracle's own automorphism: in the R x C view of a limb (C = 2^min(8,
    logN-4) words per row) X -> X^g takes every row to a single row and every
    aligned block of 8 rows onto an aligned block of 8 rows."""
    N = 1 << logN
    C = 1 << min(8, logN - 4)
    R = N // C
    idx = np.arange(N, dtype=np.uint32)
    for g in sorted({5, oracle.galois_elt(N // 2 - 1, logN), 2 * N - 1, oracle.galois_elt(3, logN) * (2 * N - 1) % (2 * N)}):
        src = oracle.automorph_ntt(idx, logN, g).astype(np.int64)  # slot k of x(X^g) is slot src[k] of x
        rows = (src // C).reshape(R, C)
        assert (rows == rows[:, :1]).all(), g                   # one source row per output row
        rho = rows[:, 0]
        assert sorted(rho.tolist()) == list(range(R)), g          # a permutation of the rows
        blocks = rho.reshape(R // 8, 8)
        assert (blocks // 8 == blocks[:, :1] // 8).all(), g       # aligned 8-blocks onto aligned 8-blocks
