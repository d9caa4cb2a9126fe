"""Pins of the oracle's baby-step giant-step linear transform.

out = sum_i rot_{gg_i}( sum_j d_{i,j} (.) rot_{gb_j}(ct) ), the diagonal
method of CKKS bootstrapping's CoeffsToSlots / SlotsToCoeffs with hoisted baby
steps (baby step 0 and giant step 0 are the identity).  It is pinned by
reductions to already pinned operations, each exact:
  - one diagonal (n1 = n2 = 1): the slot-wise product d (.) ct;
  - no giant steps (n2 = 1): sum_j d_j (.) (hoisted rotation j of ct);
  - no baby steps (n1 = 1): d_0 (.) ct + sum_i rotation_i(d_i (.) ct);
  - a single all-ones diagonal at (i, j): the giant rotation i of the hoisted
    baby rotation j (the order in which the two rotations compose);
and, with real keys, by decryption: c0' + c1' s equals the same transform
applied to the decrypted input (automorphisms and slot products, pinned
elsewhere) within sum_{i, j>=1} |d_{i,j}|_1 B_j + sum_{i>=1} B_i, where B is
the key-switching bound of one rotation key (the baby-step error is
multiplied by the diagonal in the coefficient domain, a giant step adds its
own key-switching error, and automorphisms preserve the infinity norm).
"""
import numpy as np
import pytest

from key_switching_b200 import synth
from tests import helpers as H
from tests.test_oracle_keyswitch import _bound

LOGN, L, ALPHA, BITS = 10, 5, 2, 30


def _params(oracle):
    pr = oracle.gen_primes(LOGN, BITS, L + ALPHA)
    return oracle.Params(LOGN, pr[ALPHA:], pr[:ALPHA])


def _rot_key(oracle, P, s, g, seed):
    """Seed, 'b' half and key errors of a real key for s(X^g) -> s."""
    sp = oracle.automorph(s, P.logN, g)
    e = synth.gaussian_errors(P.dnum, P.N, 500 + seed)
    kseed = synth.chacha_seed(500 + seed, g)
    return kseed, oracle.ksk_gen(P, s, sp, e, kseed), e


def _uniform_key(P, seed):
    prim = [P.prime(g) for g in range(P.L + P.alpha)]
    return synth.chacha_seed(seed, 9), np.stack([synth.uniform_residues(prim, P.N, seed, 0xB, j)
                                                 for j in range(P.dnum)])


def _ct(P, l, seed):
    return (synth.uniform_residues(P.q[:l], P.N, seed, 0), synth.uniform_residues(P.q[:l], P.N, seed, 1))


def _diag_uniform(P, l, n2, n1, seed):
    return np.stack([np.stack([synth.uniform_residues(P.q[:l], P.N, seed, i, j) for j in range(n1)])
                     for i in range(n2)])


def _slot_mul(P, l, d, x):
    return np.stack([H.mulmod(d[t], x[t], int(P.q[t])) for t in range(l)])


def _add(P, l, x, y):
    return np.stack([H.addmod(x[t], y[t], int(P.q[t])) for t in range(l)])


def test_single_diagonal_is_the_slot_product(oracle):
    P = _params(oracle)
    l = 4
    c0, c1 = _ct(P, l, 1)
    d = _diag_uniform(P, l, 1, 1, 2)
    o0, o1 = oracle.linear_transform(P, c0, c1, l, d, [], [], [], [], [], [])
    assert np.array_equal(o0, _slot_mul(P, l, d[0, 0], c0))
    assert np.array_equal(o1, _slot_mul(P, l, d[0, 0], c1))


def test_no_giant_steps_is_a_sum_of_hoisted_rotations(oracle):
    P = _params(oracle)
    l = 5
    c0, c1 = _ct(P, l, 3)
    gb = [oracle.galois_elt(1, LOGN), oracle.galois_elt(2, LOGN), 2 * P.N - 1]
    keys = [_uniform_key(P, 10 + j) for j in range(3)]
    d = _diag_uniform(P, l, 1, 4, 4)
    o0, o1 = oracle.linear_transform(P, c0, c1, l, d, gb, [k[0] for k in keys], [k[1] for k in keys], [], [], [])
    hs = oracle.rotate_hoisted(P, c0, c1, l, gb, [k[0] for k in keys], [k[1] for k in keys])
    w0, w1 = _slot_mul(P, l, d[0, 0], c0), _slot_mul(P, l, d[0, 0], c1)
    for j, (h0, h1) in enumerate(hs, start=1):
        w0 = _add(P, l, w0, _slot_mul(P, l, d[0, j], h0))
        w1 = _add(P, l, w1, _slot_mul(P, l, d[0, j], h1))
    assert np.array_equal(o0, w0) and np.array_equal(o1, w1)


def test_no_baby_steps_is_a_sum_of_rotations(oracle):
    P = _params(oracle)
    l = 3
    c0, c1 = _ct(P, l, 5)
    gg = [oracle.galois_elt(3, LOGN), oracle.galois_elt(6, LOGN)]
    keys = [_uniform_key(P, 20 + i) for i in range(2)]
    d = _diag_uniform(P, l, 3, 1, 6)
    o0, o1 = oracle.linear_transform(P, c0, c1, l, d, [], [], [], gg, [k[0] for k in keys], [k[1] for k in keys])
    w0, w1 = _slot_mul(P, l, d[0, 0], c0), _slot_mul(P, l, d[0, 0], c1)
    for i in (1, 2):
        r0, r1 = oracle.rotate(P, _slot_mul(P, l, d[i, 0], c0), _slot_mul(P, l, d[i, 0], c1), l, gg[i - 1],
                               keys[i - 1][0], keys[i - 1][1])
        w0, w1 = _add(P, l, w0, r0), _add(P, l, w1, r1)
    assert np.array_equal(o0, w0) and np.array_equal(o1, w1)


@pytest.mark.parametrize("i,j", [(2, 1), (1, 2), (0, 0), (2, 0)])
def test_one_unit_diagonal_composes_giant_after_baby(oracle, i, j):
    P = _params(oracle)
    l = 4
    c0, c1 = _ct(P, l, 7)
    gb = [oracle.galois_elt(1, LOGN), oracle.galois_elt(2, LOGN)]
    gg = [oracle.galois_elt(3, LOGN), oracle.galois_elt(6, LOGN)]
    kb = [_uniform_key(P, 30 + k) for k in range(2)]
    kg = [_uniform_key(P, 40 + k) for k in range(2)]
    d = np.zeros((3, 3, l, P.N), dtype=np.uint32)
    d[i, j] = 1  # the plaintext 1: every slot 1
    o0, o1 = oracle.linear_transform(P, c0, c1, l, d, gb, [k[0] for k in kb], [k[1] for k in kb],
                                     gg, [k[0] for k in kg], [k[1] for k in kg])
    x0, x1 = c0, c1
    if j:
        [(x0, x1)] = oracle.rotate_hoisted(P, c0, c1, l, [gb[j - 1]], [kb[j - 1][0]], [kb[j - 1][1]])
    if i:
        x0, x1 = oracle.rotate(P, x0, x1, l, gg[i - 1], kg[i - 1][0], kg[i - 1][1])
    assert np.array_equal(o0, x0) and np.array_equal(o1, x1)


def _lt_error(oracle, P, l, s, d, gb, gg, c0, c1, o0, o1):
    """max |(o0 + o1 s) - sum_i sigma_gg_i(sum_j d_ij sigma_gb_j(c0 + c1 s))| over Q_l."""
    n2, n1 = d.shape[:2]
    diffs = []
    for t in range(l):
        q = int(P.q[t])
        sh = oracle.ntt_fwd(H.reduce_signed(s, q), LOGN, q)
        m = H.addmod(c0[t], H.mulmod(c1[t], sh, q), q)   # the decrypted input, NTT domain
        want = np.zeros(P.N, dtype=np.uint32)
        for i in range(n2):
            wi = np.zeros(P.N, dtype=np.uint32)
            for j in range(n1):
                mj = m if j == 0 else oracle.automorph_ntt(m, LOGN, gb[j - 1])
                wi = H.addmod(wi, H.mulmod(d[i, j, t], mj, q), q)
            want = H.addmod(want, wi if i == 0 else oracle.automorph_ntt(wi, LOGN, gg[i - 1]), q)
        got = H.addmod(o0[t], H.mulmod(o1[t], sh, q), q)
        diffs.append(oracle.ntt_inv(H.submod(got, want, q), LOGN, q))
    Ql = H.prod(P.q[:l])
    return max(abs(int(v)) for v in H.centered(H.crt_lift(np.stack(diffs), P.q[:l]), Ql)), Ql


def test_decrypts_to_the_transformed_plaintext(oracle):
    """Real rotation keys, small diagonals: Dec(out) matches
    sum_i sigma_{gg_i}(sum_j d_ij sigma_{gb_j}(Dec(ct))) within the bound; a
    wrong giant key breaks it by far."""
    P = _params(oracle)
    l, n1, n2 = L, 3, 3
    s = synth.ternary_secret(P.N, 7)
    gb = [oracle.galois_elt(1, LOGN), oracle.galois_elt(2, LOGN)]
    gg = [oracle.galois_elt(3, LOGN), oracle.galois_elt(6, LOGN)]
    kb = [_rot_key(oracle, P, s, g, k) for k, g in enumerate(gb)]
    kg = [_rot_key(oracle, P, s, g, 10 + k) for k, g in enumerate(gg)]
    rng = np.random.default_rng(11)
    dint = np.zeros((n2, n1, P.N), dtype=np.int64)
    for i in range(n2):
        for j in range(n1):
            pos = rng.choice(P.N, size=4, replace=False)
            dint[i, j, pos] = rng.integers(-3, 4, size=4)
    d = np.stack([np.stack([np.stack([oracle.ntt_fwd(H.reduce_signed(dint[i, j], int(q)), LOGN, int(q))
                                      for q in P.q[:l]]) for j in range(n1)]) for i in range(n2)])
    c0, c1 = _ct(P, l, 8)
    o0, o1 = oracle.linear_transform(P, c0, c1, l, d, gb, [k[0] for k in kb], [k[1] for k in kb],
                                     gg, [k[0] for k in kg], [k[1] for k in kg])
    err, Ql = _lt_error(oracle, P, l, s, d, gb, gg, c0, c1, o0, o1)
    bound = sum(int(np.abs(dint[i, j]).sum()) * _bound(P, l, s, kb[j - 1][2])
                for i in range(n2) for j in range(1, n1)) + sum(_bound(P, l, s, k[2]) for k in kg)
    assert bound < Ql // 2
    assert err <= bound, (err, bound)
    # the giant keys swapped: each switches the wrong automorphism
    o0b, o1b = oracle.linear_transform(P, c0, c1, l, d, gb, [k[0] for k in kb], [k[1] for k in kb],
                                       gg, [kg[1][0], kg[0][0]], [kg[1][1], kg[0][1]])
    err_bad, _ = _lt_error(oracle, P, l, s, d, gb, gg, c0, c1, o0b, o1b)
    assert err_bad > 1000 * bound
