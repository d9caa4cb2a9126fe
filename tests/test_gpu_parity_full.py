"""GPU parity at the full workload sizes, every output against the oracle.

The kernels are instantiated per ring degree, so the small-ring tests do not
cover the N=2^16 and N=2^17 code.  Here, at N=2^16 (L=24, alpha=4, dnum=6)
and N=2^17 (L=40, alpha=5, dnum=8), every call the benchmark times is checked
element by element against the oracle on the same seeded inputs, bit-exact:
  - the key switch and the batched key switch with a stored 'a' half (the
    "stored" mode of the 16-key batch), as well as with regeneration;
  - all 16 outputs of the 16-key batch and all 4 of a hoisted call;
  - relinearisation of a ciphertext product, and a real s^2 -> s key whose
    output decrypts within the bound;
  - the separate calls pc_modup, pc_keyswitch_inner (both key modes) and
    pc_moddown, at l=24 (N=2^16) and l=23 (N=2^17).
"""
import numpy as np
import pytest

from key_switching_b200 import synth
from tests import gpu_util as G
from tests import helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def built():
    from key_switching_b200 import build
    build.build()


@pytest.fixture(scope="module")
def n16(built, oracle):
    return G.contexts(oracle, 16, 24, 4, 31)


def _stored_a(P, seed_id):
    """A uniform stored 'a' half [dnum][L+alpha][N] (any 'a' defines a key
    switch; the stored path reads it instead of regenerating)."""
    prim = [P.prime(g) for g in range(P.L + P.alpha)]
    return np.stack([synth.uniform_residues(prim, P.N, seed_id, 0xA, j) for j in range(P.dnum)])


def _ct(P, l, *tag):
    return (synth.uniform_residues(P.q[:l], P.N, *tag, 0), synth.uniform_residues(P.q[:l], P.N, *tag, 1))


def test_keyswitch_stored_a_n16(n16, oracle):
    """pc_keyswitch with a stored 'a' half at N=2^16, l=24 and l=13."""
    from key_switching_b200 import pc
    P, C = n16
    seed, b = G.random_key(P, 41)
    a = _stored_a(P, 41)
    key = pc.KSK(seed, G.dev(b), G.dev(a))
    cases = []
    for l in (24, 13):
        C.ensure_workspace(l)
        c0, c1 = _ct(P, l, 42, l)
        o0, o1 = G.filled(l, P.N), G.filled(l, P.N)
        C.keyswitch(G.dev(c0), G.dev(c1), l, key, o0, o1)
        cases.append((l, G.host(o0), G.host(o1), c0, c1))
    want = G.oracle_map(oracle, P, [(oracle.keyswitch, (P, c0, c1, l, seed, b, a)) for l, _, _, c0, c1 in cases])
    for (l, g0, g1, _, _), (w0, w1) in zip(cases, want):
        assert np.array_equal(g0, w0) and np.array_equal(g1, w1), l


@pytest.mark.parametrize("mode", ["regen", "stored"])
def test_batch16_n16_all_outputs(n16, oracle, mode):
    """16 ciphertexts under 16 distinct keys in one pc_keyswitch_batch call;
    every one of the 16 outputs against the oracle, in both key modes."""
    from key_switching_b200 import pc
    P, C = n16
    l, B = 24, 16
    C.ensure_workspace(l, B)
    keys, raw = [], []
    for k in range(B):
        seed, b = G.random_key(P, 100 + k)
        a = _stored_a(P, 100 + k) if mode == "stored" else None
        raw.append((seed, b, a))
        keys.append(pc.KSK(seed, G.dev(b), None if a is None else G.dev(a)))
    ct = np.stack([np.stack(_ct(P, l, 7, k)) for k in range(B)])
    out = G.filled(B, 2, l, P.N)
    C.keyswitch_batch(G.dev(ct), B, l, keys, out)
    got = G.host(out)
    want = G.oracle_map(oracle, P, [(oracle.keyswitch, (P, ct[k, 0], ct[k, 1], l, s, b, a))
                                    for k, (s, b, a) in enumerate(raw)])
    for k, (w0, w1) in enumerate(want):
        assert np.array_equal(got[k, 0], w0) and np.array_equal(got[k, 1], w1), k


def test_rotate_hoisted_n16_all_outputs(n16, oracle):
    """Four hoisted rotations (steps 1, 2, 4, 8) at N=2^16, l=24, each against
    the oracle's hoisted rotation."""
    from key_switching_b200 import pc
    P, C = n16
    l = 24
    C.ensure_workspace(l, 4)
    gs = [oracle.galois_elt(r, 16) for r in (1, 2, 4, 8)]
    keys = [G.random_key(P, 300 + i) for i in range(4)]
    c0, c1 = _ct(P, l, 6)
    out = G.filled(4, 2, l, P.N)
    C.rotate_hoisted(G.dev(c0), G.dev(c1), l, gs, [pc.KSK(s, G.dev(b)) for s, b in keys], out)
    got = G.host(out)
    want = G.oracle_map(oracle, P, [(oracle.rotate_hoisted, (P, c0, c1, l, [g], [s], [b]))
                                    for g, (s, b) in zip(gs, keys)])
    for i, [(w0, w1)] in enumerate(want):
        assert np.array_equal(got[i, 0], w0) and np.array_equal(got[i, 1], w1), i


def test_relinearize_n16(n16, oracle):
    """Tensor + relinearisation of two uniform ciphertexts at N=2^16, l=24 and
    l=5, and squaring at l=24."""
    from key_switching_b200 import pc
    P, C = n16
    seed, b = G.random_key(P, 13)
    key = pc.KSK(seed, G.dev(b))
    cases = []
    for l, square in ((24, False), (5, False), (24, True)):
        C.ensure_workspace(l)
        x = np.stack(_ct(P, l, 80, l))
        y = x if square else np.stack(_ct(P, l, 90, l))
        dx = G.dev(x)
        out = G.filled(2, l, P.N)
        C.relinearize(dx, dx if square else G.dev(y), l, key, out)
        cases.append((l, G.host(out), x, y))
    want = G.oracle_map(oracle, P, [(oracle.relinearize, (P, x[0], x[1], y[0], y[1], l, seed, b))
                                    for l, _, x, y in cases])
    for (l, got, _, _), (w0, w1) in zip(cases, want):
        assert np.array_equal(got[0], w0) and np.array_equal(got[1], w1), l


def test_relinearize_n16_real_key_decrypts(n16, oracle):
    """A real s^2 -> s key (Hamming-weight-192 secret) at N=2^16, l=24: the GPU
    relinearisation is bit-exact and c0' + c1' s equals d0 + d1 s + d2 s^2
    within the key-switching bound."""
    from key_switching_b200 import pc
    from tests.test_oracle_keyswitch import _bound
    P, C = n16
    s, s2, e, kseed, b = G.real_key(oracle, P, "square", 3, hw=synth.HAMMING_WEIGHT)
    l = 24
    C.ensure_workspace(l)
    x = np.stack(_ct(P, l, 71))
    y = np.stack(_ct(P, l, 72))
    out = G.filled(2, l, P.N)
    C.relinearize(G.dev(x), G.dev(y), l, pc.KSK(kseed, G.dev(b)), out)
    got = G.host(out)
    w0, w1 = oracle.relinearize(P, x[0], x[1], y[0], y[1], l, kseed, b)
    assert np.array_equal(got[0], w0) and np.array_equal(got[1], w1)
    d0, d1, d2 = oracle.tensor(P, x[0], x[1], y[0], y[1], l)
    diffs = []
    for i in range(l):
        q = int(P.q[i])
        sh = oracle.ntt_fwd(H.reduce_signed(s, q), 16, q)
        s2h = oracle.ntt_fwd(H.reduce_signed(s2, q), 16, q)
        after = H.addmod(got[0][i], H.mulmod(got[1][i], sh, q), q)
        before = H.addmod(H.addmod(d0[i], H.mulmod(d1[i], sh, q), q), H.mulmod(d2[i], s2h, q), q)
        diffs.append(oracle.ntt_inv(H.submod(after, before, q), 16, q))
    err = max(abs(int(v)) for v in H.centered(H.crt_lift(np.stack(diffs), P.q[:l]), H.prod(P.q[:l])))
    assert err <= _bound(P, l, s, e)


@pytest.mark.parametrize("shape,l", [((16, 24, 4, 31), 24), ((17, 40, 5, 31), 23)])
def test_standalone_calls_full_size(built, oracle, shape, l):
    """pc_modup, pc_keyswitch_inner (regenerated and stored 'a') and pc_moddown
    at the full ring sizes, each on its own against the oracle's step."""
    from key_switching_b200 import pc
    P, C = G.contexts(oracle, *shape)
    C.ensure_workspace(l)
    beta, ll = -(-l // P.alpha), l + P.alpha
    seed, b = G.random_key(P, 51)
    a = _stored_a(P, 51)
    c1 = synth.uniform_residues(P.q[:l], P.N, 52, l)
    accr = np.stack([synth.uniform_residues(P.level_primes(l), P.N, 53, l, h) for h in range(2)])
    want_ext, want_md = G.oracle_map(oracle, P, [(oracle.modup, (P, c1, l)), (oracle.moddown, (P, accr, l))])
    ext = G.filled(beta, ll, P.N)
    C.modup(G.dev(c1), l, ext)
    assert np.array_equal(G.host(ext), want_ext)
    de = G.dev(want_ext)
    acc_r, acc_s = G.filled(2, ll, P.N), G.filled(2, ll, P.N)
    C.keyswitch_inner(de, l, pc.KSK(seed, G.dev(b)), acc_r)
    C.keyswitch_inner(de, l, pc.KSK(seed, G.dev(b), G.dev(a)), acc_s)
    w_r, w_s = G.oracle_map(oracle, P, [(oracle.inner, (P, want_ext, l, seed, b)),
                                        (oracle.inner, (P, want_ext, l, seed, b, a))])
    assert np.array_equal(G.host(acc_r), w_r)
    assert np.array_equal(G.host(acc_s), w_s)
    out = G.filled(2, l, P.N)
    C.moddown(G.dev(accr), l, out)
    assert np.array_equal(G.host(out), want_md)
    C.check()


def test_hoisted_identity_equals_keyswitch_n16(n16, oracle):
    """A hoisted rotation by g = 1 (k_inner_rot's body) equals the plain key
    switch (the two-group inner product) bit for bit at N=2^16, l=24 and
    l=9, both with a regenerated and with a stored 'a' half: the two inner
    product texts are pinned against each other."""
    from key_switching_b200 import pc
    P, C = n16
    for l, stored in ((24, False), (9, False), (24, True)):
        C.ensure_workspace(l)
        seed, b = G.random_key(P, 61 + l)
        key = pc.KSK(seed, G.dev(b), G.dev(_stored_a(P, 61)) if stored else None)
        c0, c1 = _ct(P, l, 62, l)
        d0, d1 = G.dev(c0), G.dev(c1)
        o0, o1 = G.filled(l, P.N), G.filled(l, P.N)
        C.keyswitch(d0, d1, l, key, o0, o1)
        h = G.filled(1, 2, l, P.N)
        C.rotate_hoisted(d0, d1, l, [1], [key], h)
        got = G.host(h)
        assert np.array_equal(got[0, 0], G.host(o0)) and np.array_equal(got[0, 1], G.host(o1)), (l, stored)
