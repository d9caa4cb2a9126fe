"""GPU parity of the rotation and relinearisation paths (through the C ABI)
against the oracle, bit-exact on every limb: single rotations (automorphism
applied while the kernels read c1 and c0), hoisted rotations (one ModUp, the
automorphism applied to the extended limbs inside the inner product) and
relinearisation (tensor formed inside the kernels), at small rings with
ragged levels and at the N=2^16 workload's full size."""
import numpy as np
import pytest

from key_switching_b200 import synth
from tests import gpu_util as G
from tests import helpers as H

pytestmark = pytest.mark.gpu

SMALL = [  # (logN, L, alpha, bits)
    (10, 5, 2, 30),   # partial last digit
    (11, 7, 3, 31),
    (12, 4, 2, 30),   # the relinearisation workload's basis
    (13, 6, 4, 31),
]


@pytest.fixture(scope="module")
def built():
    from key_switching_b200 import build
    build.build()


def _galois_set(oracle, logN):
    N = 1 << logN
    return [oracle.galois_elt(1, logN), oracle.galois_elt(N // 2 - 1, logN), 2 * N - 1,
            oracle.galois_elt(3, logN) * (2 * N - 1) % (2 * N), 1]


def _ct(P, l, tag):
    return (synth.uniform_residues(P.q[:l], P.N, tag, l, 0), synth.uniform_residues(P.q[:l], P.N, tag, l, 1))


@pytest.mark.parametrize("logN,L,alpha,bits", SMALL)
def test_rotate(built, oracle, logN, L, alpha, bits):
    from key_switching_b200 import pc
    P, C = G.contexts(oracle, logN, L, alpha, bits)
    seed, b = G.random_key(P, 11)
    key = pc.KSK(seed, G.dev(b))
    for l in sorted({L, L - 1, 1}, reverse=True):
        C.ensure_workspace(l)
        c0, c1 = _ct(P, l, 40 + l)
        for g in _galois_set(oracle, logN):
            o0, o1 = G.filled(l, P.N), G.filled(l, P.N)
            C.rotate(G.dev(c0), G.dev(c1), l, g, key, o0, o1)
            w0, w1 = oracle.rotate(P, c0, c1, l, g, seed, b)
            assert np.array_equal(G.host(o0), w0), (l, g)
            assert np.array_equal(G.host(o1), w1), (l, g)
    C.check()


@pytest.mark.parametrize("logN,L,alpha,bits", SMALL)
def test_rotate_hoisted(built, oracle, logN, L, alpha, bits):
    from key_switching_b200 import pc
    P, C = G.contexts(oracle, logN, L, alpha, bits)
    gs = _galois_set(oracle, logN)
    keys = [G.random_key(P, 200 + i) for i in range(len(gs))]
    kk = [pc.KSK(s, G.dev(b)) for s, b in keys]
    for l in sorted({L, alpha + 1, 1}, reverse=True):
        C.ensure_workspace(l, len(gs))
        c0, c1 = _ct(P, l, 60 + l)
        out = G.filled(len(gs), 2, l, P.N)
        C.rotate_hoisted(G.dev(c0), G.dev(c1), l, gs, kk, out)
        got = G.host(out)
        want = oracle.rotate_hoisted(P, c0, c1, l, gs, [s for s, _ in keys], [b for _, b in keys])
        for i, (w0, w1) in enumerate(want):
            assert np.array_equal(got[i, 0], w0), (l, gs[i])
            assert np.array_equal(got[i, 1], w1), (l, gs[i])
    C.check()


def test_rotate_hoisted_more_than_one_batch(built, oracle):
    """18 hoisted rotations: two launch batches (16 + 2) over one ModUp, each
    rotation bit-exact with the oracle, l below L."""
    from key_switching_b200 import pc
    P, C = G.contexts(oracle, 10, 5, 2, 30)
    N = P.N
    gs = [pow(5, r, 2 * N) for r in range(1, 19)]
    keys = [G.random_key(P, 600 + i) for i in range(len(gs))]
    kk = [pc.KSK(s, G.dev(b)) for s, b in keys]
    l = 4
    C.ensure_workspace(l, 16)
    c0, c1 = _ct(P, l, 70)
    out = G.filled(len(gs), 2, l, N)
    C.rotate_hoisted(G.dev(c0), G.dev(c1), l, gs, kk, out)
    got = G.host(out)
    want = oracle.rotate_hoisted(P, c0, c1, l, gs, [s for s, _ in keys], [b for _, b in keys])
    for i, (w0, w1) in enumerate(want):
        assert np.array_equal(got[i, 0], w0) and np.array_equal(got[i, 1], w1), i
    C.check()


def test_rotate_n17_low_level(built, oracle):
    """N=2^17, L=40, alpha=5 (the level-sweep basis) at l=7: a single and two
    hoisted rotations, bit-exact."""
    from key_switching_b200 import pc
    P, C = G.contexts(oracle, 17, 40, 5, 31)
    l = 7
    C.ensure_workspace(l, 2)
    seed, b = G.random_key(P, 17)
    key = pc.KSK(seed, G.dev(b))
    c0, c1 = _ct(P, l, 80)
    g = oracle.galois_elt(3, 17)
    o0, o1 = G.filled(l, P.N), G.filled(l, P.N)
    C.rotate(G.dev(c0), G.dev(c1), l, g, key, o0, o1)
    w0, w1 = oracle.rotate(P, c0, c1, l, g, seed, b)
    assert np.array_equal(G.host(o0), w0) and np.array_equal(G.host(o1), w1)
    gs = [g, 2 * P.N - 1]
    out = G.filled(2, 2, l, P.N)
    C.rotate_hoisted(G.dev(c0), G.dev(c1), l, gs, [key, key], out)
    got = G.host(out)
    for i, (h0, h1) in enumerate(oracle.rotate_hoisted(P, c0, c1, l, gs, [seed, seed], [b, b])):
        assert np.array_equal(got[i, 0], h0) and np.array_equal(got[i, 1], h1), i


@pytest.mark.parametrize("logN,L,alpha,bits", SMALL)
def test_relinearize(built, oracle, logN, L, alpha, bits):
    from key_switching_b200 import pc
    P, C = G.contexts(oracle, logN, L, alpha, bits)
    seed, b = G.random_key(P, 13)
    key = pc.KSK(seed, G.dev(b))
    for l in sorted({L, 2, 1}, reverse=True):
        C.ensure_workspace(l)
        x = np.stack(_ct(P, l, 80 + l))
        y = np.stack(_ct(P, l, 90 + l))
        for yy in (y, x):  # product and square
            out = G.filled(2, l, P.N)
            dx = G.dev(x)
            C.relinearize(dx, dx if yy is x else G.dev(yy), l, key, out)
            w0, w1 = oracle.relinearize(P, x[0], x[1], yy[0], yy[1], l, seed, b)
            got = G.host(out)
            assert np.array_equal(got[0], w0), l
            assert np.array_equal(got[1], w1), l
    C.check()


def _decrypt_rot_error(oracle, P, l, s, g, c0, c1, o0, o1):
    sg = oracle.automorph(s, P.logN, g)
    diffs = []
    for i in range(l):
        q = int(P.q[i])
        sh = oracle.ntt_fwd(H.reduce_signed(s, q), P.logN, q)
        sgh = oracle.ntt_fwd(H.reduce_signed(sg, q), P.logN, q)
        after = H.addmod(o0[i], H.mulmod(o1[i], sh, q), q)
        before = H.addmod(oracle.automorph_ntt(c0[i], P.logN, g),
                          H.mulmod(oracle.automorph_ntt(c1[i], P.logN, g), sgh, q), q)
        diffs.append(oracle.ntt_inv(H.submod(after, before, q), P.logN, q))
    Ql = H.prod(P.q[:l])
    return max(abs(int(v)) for v in H.centered(H.crt_lift(np.stack(diffs), P.q[:l]), Ql))


def test_rotate_n16_full_size_real_key(built, oracle):
    """N=2^16, L=24, alpha=4, the rotation-by-1 key at the top level: every
    limb bit-exact, and the GPU result decrypts to the rotated plaintext."""
    from key_switching_b200 import pc
    from tests.test_oracle_keyswitch import _bound
    P, C = G.contexts(oracle, 16, 24, 4, 31)
    s, sp, e, kseed, b = G.real_key(oracle, P, "rot", 0, r=1, hw=synth.HAMMING_WEIGHT)
    g = oracle.galois_elt(1, 16)
    l = 24
    C.ensure_workspace(l)
    c0, c1 = _ct(P, l, 5)
    o0, o1 = G.filled(l, P.N), G.filled(l, P.N)
    C.rotate(G.dev(c0), G.dev(c1), l, g, pc.KSK(kseed, G.dev(b)), o0, o1)
    g0, g1 = G.host(o0), G.host(o1)
    w0, w1 = oracle.rotate(P, c0, c1, l, g, kseed, b)
    assert np.array_equal(g0, w0) and np.array_equal(g1, w1)
    assert _decrypt_rot_error(oracle, P, l, s, g, c0, c1, g0, g1) <= _bound(P, l, s, e)


def test_relinearize_n12_real_key_decrypts(built, oracle):
    """The N=2^12, L=4, alpha=2 s^2 -> s key on a product of two ciphertexts:
    bit-exact, and c0' + c1' s matches d0 + d1 s + d2 s^2 within the bound."""
    from key_switching_b200 import pc
    from tests.test_oracle_keyswitch import _bound
    P, C = G.contexts(oracle, 12, 4, 2, 30)
    s, s2, e, kseed, b = G.real_key(oracle, P, "square", 0)
    l = 4
    C.ensure_workspace(l)
    x = np.stack(_ct(P, l, 7))
    y = np.stack(_ct(P, l, 8))
    out = G.filled(2, l, P.N)
    C.relinearize(G.dev(x), G.dev(y), l, pc.KSK(kseed, G.dev(b)), out)
    got = G.host(out)
    w0, w1 = oracle.relinearize(P, x[0], x[1], y[0], y[1], l, kseed, b)
    assert np.array_equal(got[0], w0) and np.array_equal(got[1], w1)
    d0, d1, d2 = oracle.tensor(P, x[0], x[1], y[0], y[1], l)
    diffs = []
    for i in range(l):
        q = int(P.q[i])
        sh = oracle.ntt_fwd(H.reduce_signed(s, q), 12, q)
        s2h = oracle.ntt_fwd(H.reduce_signed(s2, q), 12, q)
        after = H.addmod(got[0][i], H.mulmod(got[1][i], sh, q), q)
        before = H.addmod(H.addmod(d0[i], H.mulmod(d1[i], sh, q), q), H.mulmod(d2[i], s2h, q), q)
        diffs.append(oracle.ntt_inv(H.submod(after, before, q), 12, q))
    Ql = H.prod(P.q)
    err = max(abs(int(v)) for v in H.centered(H.crt_lift(np.stack(diffs), P.q), Ql))
    assert err <= _bound(P, l, s, e)


def test_rotation_error_paths(built, oracle):
    from key_switching_b200 import pc
    P, C = G.contexts(oracle, 12, 4, 2, 30)
    seed, b = G.random_key(P, 5)
    key = pc.KSK(seed, G.dev(b))
    C.ensure_workspace(4)
    c0, c1 = G.empty(4, P.N), G.empty(4, P.N)
    o0, o1 = G.empty(4, P.N), G.empty(4, P.N)
    for g in (0, 4, 2 * P.N + 1, 4 * P.N - 1):  # even or beyond 2N
        with pytest.raises(pc.PCError) as ei:
            C.rotate(c0, c1, 4, g, key, o0, o1)
        assert ei.value.code == -1, g
    with pytest.raises(pc.PCError) as ei:
        C.rotate(c0, c1, 4, 5, key, c0, o1)  # in place is refused
    assert ei.value.code == -1
    out = G.empty(2, 2, 4, P.N)
    with pytest.raises(pc.PCError) as ei:
        C.rotate_hoisted(out[1, 0], c1, 4, [5, 25], [key, key], out)  # c0 inside out
    assert ei.value.code == -1
    with pytest.raises(pc.PCError) as ei:
        C.rotate_hoisted(c0, c1, 4, [5, 6], [key, key], out)
    assert ei.value.code == -1
    with pytest.raises(pc.PCError) as ei:  # two rotations need two slices of workspace
        C.rotate_hoisted(c0, c1, 4, [5, 25], [key, key], out)
    assert ei.value.code == -7
    C.ensure_workspace(4, 2)
    with pytest.raises(pc.PCError) as ei:  # no rotation at all
        C.rotate_hoisted(c0, c1, 4, [], [], out)
    assert ei.value.code == -1
    with pytest.raises(pc.PCError) as ei:  # no ciphertext at all
        C.keyswitch_batch(out, 0, 4, [], out)
    assert ei.value.code == -1
    with pytest.raises(pc.PCError) as ei:
        C.keyswitch_host(np.zeros((1, 2, 4, P.N), dtype=np.uint32), 0, 4, [],
                         np.zeros((1, 2, 4, P.N), dtype=np.uint32))
    assert ei.value.code == -1
    x = G.empty(2, 4, P.N)
    with pytest.raises(pc.PCError) as ei:
        C.relinearize(x, x, 4, key, x)
    assert ei.value.code == -1
    with pytest.raises(pc.PCError) as ei:
        C.relinearize(x, x, 5, key, out[0])  # level above L
    assert ei.value.code == -1
    C.check()
