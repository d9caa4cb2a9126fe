"""GPU parity: every libpc call (through the C ABI) against the oracle,
bit-exact on every limb.  Sizes span several tiles and the partial last digit;
the N=2^16 / 2^17 workload shapes run at full size."""
import numpy as np
import pytest

from key_switching_b200 import synth
from tests import gpu_util as G

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


@pytest.mark.parametrize("logN,L,alpha,bits", SMALL + [(16, 24, 4, 31), (17, 40, 5, 31)])
def test_ntt_roundtrip_and_oracle(built, oracle, logN, L, alpha, bits):
    P, C = G.contexts(oracle, logN, L, alpha, bits)
    NP = L + alpha
    batch = 2
    x = np.stack([synth.uniform_residues([P.prime(g) for g in range(NP)], P.N, 5, b) for b in range(batch)])
    d = G.dev(x)
    C.ntt_fwd(d, 0, NP, batch)
    f = G.host(d)
    # oracle on a sample of limbs (all limbs for the small rings)
    limbs = range(NP) if logN <= 13 else [0, 1, L - 1, L, NP - 1]
    for b in range(batch):
        for g in limbs:
            assert np.array_equal(f[b, g], oracle.ntt_fwd(x[b, g], logN, P.prime(g))), (b, g)
    assert all(int(f[0, g].max()) < P.prime(g) for g in range(NP))
    C.ntt_inv(d, 0, NP, batch)
    assert np.array_equal(G.host(d), x)
    # inverse alone against the oracle, offset first prime
    y = G.dev(x[0, 1:3])
    C.ntt_inv(y, 1, 2, 1)
    yh = G.host(y)
    for k in range(2):
        assert np.array_equal(yh[k], oracle.ntt_inv(x[0, 1 + k], logN, P.prime(1 + k)))


@pytest.mark.parametrize("logN,L,alpha,bits", SMALL + [(16, 24, 4, 31)])
def test_psi_matches_oracle(built, oracle, logN, L, alpha, bits):
    P, C = G.contexts(oracle, logN, L, alpha, bits)
    for g in range(L + alpha):
        assert C.psi(g) == oracle.min_psi(P.prime(g), logN)


@pytest.mark.parametrize("logN,L,alpha,bits,l", [(10, 5, 2, 30, 5), (10, 5, 2, 30, 2), (16, 24, 4, 31, 24),
                                                   (17, 40, 5, 31, 7)])
def test_expand_a(built, oracle, logN, L, alpha, bits, l):
    P, C = G.contexts(oracle, logN, L, alpha, bits)
    seed = synth.chacha_seed(3, 1)
    beta = -(-l // alpha)
    out = G.filled(beta, l + alpha, P.N)
    C.expand_a(seed, l, out)
    got = G.host(out)
    pairs = [(j, t) for j in range(beta) for t in range(l + alpha)]
    if logN >= 16:
        pairs = [pairs[0], pairs[1], pairs[len(pairs) // 2], pairs[-1]]
    for j, t in pairs:
        g = P.glob(l, t)
        assert np.array_equal(got[j, t], oracle.expand_a(seed, j, g, P.prime(g), logN)), (j, t)


def _levels(L, alpha):
    return sorted({L, L - 1, alpha + 1, alpha, 1, max(1, L // 2)}, reverse=True)


@pytest.mark.parametrize("logN,L,alpha,bits", SMALL)
def test_modup_inner_moddown_stepwise(built, oracle, logN, L, alpha, bits):
    P, C = G.contexts(oracle, logN, L, alpha, bits)
    seed, b = G.random_key(P, 1)
    bd = G.dev(b)
    a_st = np.stack([np.stack([oracle.expand_a(seed, j, g, P.prime(g), logN) for g in range(L + alpha)])
                     for j in range(P.dnum)])
    ad = G.dev(a_st)
    from key_switching_b200 import pc
    for l in _levels(L, alpha):
        C.ensure_workspace(l)
        beta = -(-l // alpha)
        ll = l + alpha
        c1 = synth.uniform_residues(P.q[:l], P.N, 11, l)
        ext = G.filled(beta, ll, P.N)
        C.modup(G.dev(c1), l, ext)
        ext_h = G.host(ext)
        want_ext = oracle.modup(P, c1, l)
        assert np.array_equal(ext_h, want_ext), l
        # inner product on the oracle's ext, regenerated and stored 'a'
        acc = G.filled(2, ll, P.N)
        C.keyswitch_inner(G.dev(want_ext), l, pc.KSK(seed, bd), acc)
        want_acc = oracle.inner(P, want_ext, l, seed, b)
        assert np.array_equal(G.host(acc), want_acc), l
        acc2 = G.filled(2, ll, P.N)
        C.keyswitch_inner(G.dev(want_ext), l, pc.KSK(seed, bd, ad), acc2)
        assert np.array_equal(G.host(acc2), want_acc), l
        # ModDown on a uniform accumulator
        accr = np.stack([synth.uniform_residues(P.level_primes(l), P.N, 12, l, h) for h in range(2)])
        out = G.filled(2, l, P.N)
        C.moddown(G.dev(accr), l, out)
        assert np.array_equal(G.host(out), oracle.moddown(P, accr, l)), l


@pytest.mark.parametrize("logN,L,alpha,bits", SMALL)
def test_keyswitch_all_levels(built, oracle, logN, L, alpha, bits):
    P, C = G.contexts(oracle, logN, L, alpha, bits)
    seed, b = G.random_key(P, 2)
    from key_switching_b200 import pc
    key = pc.KSK(seed, G.dev(b))
    for l in range(L, 0, -1):
        C.ensure_workspace(l)
        c0 = synth.uniform_residues(P.q[:l], P.N, 21, l)
        c1 = synth.uniform_residues(P.q[:l], P.N, 22, l)
        o0, o1 = G.filled(l, P.N), G.filled(l, P.N)
        C.keyswitch(G.dev(c0), G.dev(c1), l, key, o0, o1)
        w0, w1 = oracle.keyswitch(P, c0, c1, l, seed, b)
        assert np.array_equal(G.host(o0), w0), l
        assert np.array_equal(G.host(o1), w1), l
    C.check()


def test_keyswitch_in_place_and_stored_a(built, oracle):
    P, C = G.contexts(oracle, 12, 4, 2, 30)
    seed, b = G.random_key(P, 4)
    a_st = np.stack([np.stack([oracle.expand_a(seed, j, g, P.prime(g), 12) for g in range(P.L + P.alpha)])
                     for j in range(P.dnum)])
    from key_switching_b200 import pc
    l = 4
    C.ensure_workspace(l)
    c0 = synth.uniform_residues(P.q[:l], P.N, 31)
    c1 = synth.uniform_residues(P.q[:l], P.N, 32)
    w0, w1 = oracle.keyswitch(P, c0, c1, l, seed, b)
    d0, d1 = G.dev(c0), G.dev(c1)
    C.keyswitch(d0, d1, l, pc.KSK(seed, G.dev(b), G.dev(a_st)), d0, d1)
    assert np.array_equal(G.host(d0), w0) and np.array_equal(G.host(d1), w1)


def test_relinearisation_n12_real_key_decrypts(built, oracle):
    """The N=2^12, L=4, alpha=2 s^2 -> s workload with a real key: bit-exact,
    and the GPU output decrypts under s."""
    from key_switching_b200 import pc
    from tests.test_oracle_keyswitch import _bound
    from tests import helpers as H
    P, C = G.contexts(oracle, 12, 4, 2, 30)
    s, sp, e, kseed, b = G.real_key(oracle, P, "square", 0)
    l = 4
    C.ensure_workspace(l)
    c0 = synth.uniform_residues(P.q, P.N, 0, 0)
    c1 = synth.uniform_residues(P.q, P.N, 0, 1)
    o0, o1 = G.empty(l, P.N), G.empty(l, P.N)
    C.keyswitch(G.dev(c0), G.dev(c1), l, pc.KSK(kseed, G.dev(b)), o0, o1)
    g0, g1 = G.host(o0), G.host(o1)
    w0, w1 = oracle.keyswitch(P, c0, c1, l, kseed, b)
    assert np.array_equal(g0, w0) and np.array_equal(g1, w1)
    diffs = []
    for i in range(l):
        q = int(P.q[i])
        sh = oracle.ntt_fwd(H.reduce_signed(s, q), 12, q)
        sph = oracle.ntt_fwd(H.reduce_signed(sp, q), 12, q)
        diffs.append(oracle.ntt_inv(H.submod(H.addmod(g0[i], H.mulmod(g1[i], sh, q), q),
                                             H.addmod(c0[i], H.mulmod(c1[i], sph, q), q), q), 12, q))
    Ql = H.prod(P.q)
    err = H.centered(H.crt_lift(np.stack(diffs), P.q), Ql)
    assert max(abs(int(v)) for v in err) <= _bound(P, l, s, e)


def test_rotation_n16_full_size(built, oracle):
    """N=2^16, L=24, alpha=4, dnum=6, rotation-by-1 key, top level: the bench's
    single-ciphertext workload in the same launch configuration, every limb."""
    from key_switching_b200 import pc
    P, C = G.contexts(oracle, 16, 24, 4, 31)
    s, sp, e, kseed, b = G.real_key(oracle, P, "rot", 0, r=1, hw=synth.HAMMING_WEIGHT)
    l = 24
    C.ensure_workspace(l)
    c0 = synth.uniform_residues(P.q, P.N, 1, 0)
    c1 = synth.uniform_residues(P.q, P.N, 1, 1)
    o0, o1 = G.empty(l, P.N), G.empty(l, P.N)
    C.keyswitch(G.dev(c0), G.dev(c1), l, pc.KSK(kseed, G.dev(b)), o0, o1)
    w0, w1 = oracle.keyswitch(P, c0, c1, l, kseed, b)
    assert np.array_equal(G.host(o0), w0) and np.array_equal(G.host(o1), w1)


def test_batch_more_than_one_launch(built, oracle):
    """20 ciphertexts with 20 keys: the inner product runs in two launches of
    16 + 4 keys; every ciphertext bit-exact with the oracle (small ring)."""
    from key_switching_b200 import pc
    P, C = G.contexts(oracle, 11, 7, 3, 31)
    l, B = 6, 20
    C.ensure_workspace(l, B)
    keys, bs = [], []
    for k in range(B):
        seed, b = G.random_key(P, 700 + k)
        bs.append(b)
        keys.append(pc.KSK(seed, G.dev(b)))
    ct = np.stack([np.stack([synth.uniform_residues(P.q[:l], P.N, 8, k, h) for h in range(2)]) for k in range(B)])
    out = G.filled(B, 2, l, P.N)
    C.keyswitch_batch(G.dev(ct), B, l, keys, out)
    got = G.host(out)
    for k in range(B):
        w0, w1 = oracle.keyswitch(P, ct[k, 0], ct[k, 1], l, keys[k].seed, bs[k])
        assert np.array_equal(got[k, 0], w0) and np.array_equal(got[k, 1], w1), k


@pytest.mark.parametrize("l", [40, 23, 6, 1])
def test_sweep_n17_levels(built, oracle, l):
    """N=2^17, L=40, alpha=5, dnum=8 at sampled levels of the 40..1 sweep."""
    from key_switching_b200 import pc
    P, C = G.contexts(oracle, 17, 40, 5, 31)
    seed, b = G.random_key(P, 9)
    C.ensure_workspace(l)
    c0 = synth.uniform_residues(P.q[:l], P.N, 17, l, 0)
    c1 = synth.uniform_residues(P.q[:l], P.N, 17, l, 1)
    o0, o1 = G.empty(l, P.N), G.empty(l, P.N)
    C.keyswitch(G.dev(c0), G.dev(c1), l, pc.KSK(seed, G.dev(b)), o0, o1)
    w0, w1 = oracle.keyswitch(P, c0, c1, l, seed, b)
    assert np.array_equal(G.host(o0), w0) and np.array_equal(G.host(o1), w1)


def test_error_paths(built, oracle):
    from key_switching_b200 import pc
    P, C = G.contexts(oracle, 12, 4, 2, 30)
    seed, b = G.random_key(P, 5)
    key = pc.KSK(seed, G.dev(b))
    c = G.empty(4, P.N)
    C.set_workspace(None)
    with pytest.raises(pc.PCError) as ei:
        C.keyswitch(c, c, 4, key, c, c)
    assert ei.value.code == -7
    C.ensure_workspace(4)
    with pytest.raises(pc.PCError) as ei:
        C.keyswitch(c, c, 5, key, c, c)  # level above L
    assert ei.value.code == -1
    with pytest.raises(pc.PCError) as ei:
        C.keyswitch(c.view(-1)[1:].data_ptr(), c, 4, key, c, c)  # misaligned
    assert ei.value.code == -2
    with pytest.raises(pc.PCError) as ei:
        C.ntt_fwd(c, 5, 2)  # primes beyond the basis
    assert ei.value.code == -1
    C.check()


def test_input_checks_set_the_device_error_word(built, oracle):
    """With PC_CHECK_INPUTS, a residue not below its prime in a ciphertext or
    a key half sets the device error word (pc_check -> PC_E_DEVICE, word
    bit PC_ERR_INPUT / PC_ERR_KEY); valid inputs leave it clear; without the
    flag nothing is checked."""
    from key_switching_b200 import pc
    P, C = G.contexts(oracle, 12, 4, 2, 30)
    l = 4
    C.ensure_workspace(l)
    seed, b = G.random_key(P, 61)
    c0 = synth.uniform_residues(P.q[:l], P.N, 62, 0)
    c1 = synth.uniform_residues(P.q[:l], P.N, 62, 1)
    o0, o1 = G.empty(l, P.N), G.empty(l, P.N)
    good = pc.KSK(seed, G.dev(b))
    C.set_checks(pc.CHECK_INPUTS)
    C.keyswitch(G.dev(c0), G.dev(c1), l, good, o0, o1)
    C.check()                                   # valid inputs: word clear
    w0, w1 = oracle.keyswitch(P, c0, c1, l, seed, b)
    assert np.array_equal(G.host(o0), w0) and np.array_equal(G.host(o1), w1)
    bad1 = c1.copy()
    bad1[3, 1000] = 0xFFFFFFFF
    C.keyswitch(G.dev(c0), G.dev(bad1), l, good, o0, o1)
    with pytest.raises(pc.PCError) as ei:
        C.check()
    assert ei.value.code == -4 and C.last_error_word() == pc.ERR_INPUT
    C.check()                                   # cleared by the previous check
    bb = b.copy()
    bb[1, P.L + 1, 7] = int(P.prime(P.L + 1))   # equal to its prime: not canonical
    C.keyswitch(G.dev(c0), G.dev(c1), l, pc.KSK(seed, G.dev(bb)), o0, o1)
    with pytest.raises(pc.PCError) as ei:
        C.check()
    assert ei.value.code == -4 and C.last_error_word() == pc.ERR_KEY
    x = G.dev(np.stack([bad1] * 2))
    C.ntt_fwd(x, 0, l, 2)
    with pytest.raises(pc.PCError):
        C.check()
    C.set_checks(0)
    C.keyswitch(G.dev(c0), G.dev(bad1), l, good, o0, o1)
    C.check()                                   # not checked when off
    with pytest.raises(pc.PCError) as ei:
        C.set_checks(4)
    assert ei.value.code == -1
