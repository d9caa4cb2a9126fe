"""GPU parity of the baby-step giant-step linear transform (pc_linear_transform,
through the C ABI) against the oracle, bit-exact on every limb: small rings
with ragged levels and partial digits, more than one launch batch of hoisted
baby steps, the degenerate shapes (one diagonal, no baby steps, no giant
steps), and sampled levels of the N=2^17, L=40, alpha=5 basis."""
import numpy as np
import pytest

from key_switching_b200 import synth
from tests import gpu_util as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def built():
    from key_switching_b200 import build
    build.build()


def _case(oracle, P, l, n1, n2, tag):
    """Inputs of one transform: ciphertext, diagonals, rotation steps and keys."""
    N = P.N
    c0 = synth.uniform_residues(P.q[:l], N, tag, 0)
    c1 = synth.uniform_residues(P.q[:l], N, tag, 1)
    diag = np.stack([np.stack([synth.uniform_residues(P.q[:l], N, tag, 2, i, j) for j in range(n1)])
                     for i in range(n2)])
    gb = [pow(5, j, 2 * N) for j in range(1, n1)]                 # rotations by 1 .. n1-1
    gg = [pow(5, n1 * i, 2 * N) for i in range(1, n2)]            # rotations by n1, 2 n1, ...
    kb = [G.random_key(P, 1000 * tag + j) for j in range(n1 - 1)]
    kg = [G.random_key(P, 1000 * tag + 500 + i) for i in range(n2 - 1)]
    return c0, c1, diag, gb, gg, kb, kg


def _run(oracle, P, C, l, n1, n2, tag):
    from key_switching_b200 import pc
    c0, c1, diag, gb, gg, kb, kg = _case(oracle, P, l, n1, n2, tag)
    C.ensure_linear_transform_workspace(l, n1)
    out = G.filled(2, l, P.N)
    C.linear_transform(G.dev(c0), G.dev(c1), l, G.dev(diag), gb, [pc.KSK(s, G.dev(b)) for s, b in kb],
                       gg, [pc.KSK(s, G.dev(b)) for s, b in kg], out)
    got = G.host(out)
    w0, w1 = oracle.linear_transform(P, c0, c1, l, diag, gb, [s for s, _ in kb], [b for _, b in kb],
                                     gg, [s for s, _ in kg], [b for _, b in kg])
    assert np.array_equal(got[0], w0), (l, n1, n2)
    assert np.array_equal(got[1], w1), (l, n1, n2)


@pytest.mark.parametrize("logN,L,alpha,bits", [(10, 5, 2, 30), (11, 7, 3, 31), (12, 4, 2, 30), (13, 6, 4, 31)])
@pytest.mark.parametrize("n1,n2", [(3, 3), (4, 2), (1, 1), (1, 3), (3, 1)])
def test_linear_transform_small(built, oracle, logN, L, alpha, bits, n1, n2):
    P, C = G.contexts(oracle, logN, L, alpha, bits)
    for l in sorted({L, alpha + 1, 1}, reverse=True):
        _run(oracle, P, C, l, n1, n2, 7 + l)
    C.check()


def test_linear_transform_two_baby_batches(built, oracle):
    """18 baby steps: the hoisted rotations run in two launch batches (16 + 1)."""
    P, C = G.contexts(oracle, 10, 5, 2, 30)
    _run(oracle, P, C, 4, 18, 2, 3)


@pytest.mark.parametrize("l,n1,n2", [(23, 3, 3), (5, 4, 4), (40, 2, 2)])
def test_linear_transform_n17_levels(built, oracle, l, n1, n2):
    """N=2^17, L=40, alpha=5, dnum=8 at sampled levels of the sweep: the
    bench's 4 x 4 shape at a low level, the top level with 2 x 2."""
    P, C = G.contexts(oracle, 17, 40, 5, 31)
    _run(oracle, P, C, l, n1, n2, 40 + l)


def test_linear_transform_errors(built, oracle):
    from key_switching_b200 import pc
    P, C = G.contexts(oracle, 12, 4, 2, 30)
    l = 4
    c0, c1, diag, gb, gg, kb, kg = _case(oracle, P, l, 2, 2, 1)
    kk = [pc.KSK(s, G.dev(b)) for s, b in kb]
    kgk = [pc.KSK(s, G.dev(b)) for s, b in kg]
    d0, d1, dd = G.dev(c0), G.dev(c1), G.dev(diag)
    out = G.empty(2, l, P.N)
    C.set_workspace(None)
    with pytest.raises(pc.PCError) as ei:
        C.linear_transform(d0, d1, l, dd, gb, kk, gg, kgk, out)
    assert ei.value.code == -7
    C.ensure_linear_transform_workspace(l, 2)
    with pytest.raises(pc.PCError) as ei:
        C.linear_transform(d0, d1, l, dd, [4], kk, gg, kgk, out)      # even Galois element
    assert ei.value.code == -1
    with pytest.raises(pc.PCError) as ei:
        C.linear_transform(d0, d1, l, dd, gb, kk, gg, kgk, dd[0])     # out inside the diagonals
    assert ei.value.code == -1
    C.check()
